// Log-sum-exp merge of the aggregation's split partials into V_A (used after
// both the tensor-core and the SIMT aggregation).
#pragma once

#include "common.cuh"

namespace aa {

// ------------------------------------------------------------------ merge
// V_A = sum_s 2^(m_s - M) U_s / sum_s 2^(m_s - M) l_s.  One thread per
// (slice, agent row, 4-column group): it loads the row's (m_s, l_s) and its
// four columns of every split's U at once (the loads are independent, so one
// trip to memory), then combines them.  Up to kMergeUnroll splits per pass.
constexpr int kMergeUnroll = 16;
constexpr int kMergeThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) agent_merge_kernel(
    const float* __restrict__ part_u, const float* __restrict__ part_ml, SplitPlan plan,
    long long BH, int n_agents, int d, float* __restrict__ va_f32, T* __restrict__ va_lowp,
    float* __restrict__ ml_out = nullptr) {
  const int quads = d >> 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (idx >= BH * n_agents * quads) return;
  const int cq = (int)(idx % quads);
  const long long row = idx / quads;              // bh * n_agents + j
  const long long bh = row / n_agents;
  const int j = (int)(row % n_agents);
  const int n_splits = splits_of_slice(plan, bh);
  const long long slot0 = bh * plan.slots;
  const long long split_stride = (long long)n_agents;      // rows between consecutive splits
  const float* ml0 = part_ml + ((slot0)*n_agents + j) * 2;
  const float* u0 = part_u + ((slot0)*n_agents + j) * (long long)d + cq * 4;
  // One pass over the splits, kMergeUnroll at a time: every load of a batch
  // (running max, running sum and 4 accumulator columns of each split) is in
  // flight together; the batch's maximum rescales what was combined so far.
  float mx = -INFINITY, den = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n_splits; s0 += kMergeUnroll) {
    float2 ml[kMergeUnroll];
    float4 u[kMergeUnroll];
#pragma unroll
    for (int a = 0; a < kMergeUnroll; ++a) {
      const bool ok = s0 + a < n_splits;
      ml[a] = ok ? __ldg(reinterpret_cast<const float2*>(ml0 + (s0 + a) * split_stride * 2))
                 : make_float2(-INFINITY, 0.f);
      u[a] = ok ? __ldg(reinterpret_cast<const float4*>(u0 + (s0 + a) * split_stride * d))
                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mb = mx;
#pragma unroll
    for (int a = 0; a < kMergeUnroll; ++a) mb = fmaxf(mb, ml[a].x);
    const float r = (mx == -INFINITY) ? 0.f : exp2f(mx - mb);   // rescale of earlier batches
    den *= r;
    acc.x *= r;
    acc.y *= r;
    acc.z *= r;
    acc.w *= r;
    mx = mb;
#pragma unroll
    for (int a = 0; a < kMergeUnroll; ++a) {
      const float w = (s0 + a < n_splits) ? exp2f(ml[a].x - mx) : 0.f;
      den = fmaf(w, ml[a].y, den);
      acc.x = fmaf(w, u[a].x, acc.x);
      acc.y = fmaf(w, u[a].y, acc.y);
      acc.z = fmaf(w, u[a].z, acc.z);
      acc.w = fmaf(w, u[a].w, acc.w);
    }
  }
  const float inv = 1.f / den;
  if (ml_out != nullptr && cq == 0) {     // the row's softmax max (log2 units) and sum
    ml_out[row * 2] = mx;
    ml_out[row * 2 + 1] = den;
  }
  const float v[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  const long long o = row * d + cq * 4;
  if (va_f32) *reinterpret_cast<float4*>(va_f32 + o) = make_float4(v[0], v[1], v[2], v[3]);
  if (va_lowp) {
#pragma unroll
    for (int i = 0; i < 4; ++i) va_lowp[o + i] = from_f32<T>(v[i]);
  }
}

}  // namespace aa
