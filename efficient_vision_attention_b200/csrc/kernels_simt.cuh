// SIMT (CUDA-core, fp32-accumulate) kernels of the Agent Attention forward pass:
//   agent_pool_kernel     adaptive average pooling of Q into agents
//   simt_attend_kernel    one online-softmax attention of a block of rows over a
//                         range of columns; serves both the aggregation
//                         (rows = agents, columns = keys, split over keys,
//                         partial output) and the broadcast (rows = queries,
//                         columns = agents, normalised output)
//   agent_merge_kernel    log-sum-exp merge of the aggregation splits into V_A
// These carry the fp32 path end to end (exact enough for a 1e-5 tolerance) and
// the bf16 path for head dims the tensor-core kernels do not take.
#pragma once

#include "common.cuh"

namespace aa {

// ----------------------------------------------------------------- pooling
// One CTA per (slice bh, agent row py).  Work item = (px, 8-channel group);
// the bin's grid rows are spread over up to kPoolThreads / items threads, each
// summing its rows' bin columns with 16-byte loads, eight in flight, and the
// row partials are reduced through shared memory.  Small CTAs (4 per SM) keep
// every CTA of the usual shapes resident at once.  Sums are fp32; the divisor
// is the bin's own token count.  Writes fp32 and/or low-precision agents.
constexpr int kPoolThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kPoolThreads, 4) agent_pool_kernel(const T* __restrict__ q,
                                                                  float* __restrict__ a_f32,
                                                                  T* __restrict__ a_lowp, int N,
                                                                  int d, int grid_h, int grid_w,
                                                                  int pool_h, int pool_w) {
  __shared__ float red[kPoolThreads * 8];
  const int py = blockIdx.x;
  const long long bh = blockIdx.y;
  const int y0 = bin_start(py, grid_h, pool_h), y1 = bin_end(py, grid_h, pool_h);
  const int groups = d >> 3;
  const int items = pool_w * groups;
  const int rows = y1 - y0;
  int ysplit = (int)blockDim.x / items;
  if (ysplit < 1) ysplit = 1;
  if (ysplit > rows) ysplit = rows;
  const T* qs = q + bh * (long long)N * d;
  const long long n_agents = (long long)pool_h * pool_w;

  for (int base = 0; base < items * ysplit; base += blockDim.x) {
    const int t = base + threadIdx.x;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    int item = -1, ys = 0;
    if (t < items * ysplit) {
      item = t % items;
      ys = t / items;
      const int px = item / groups, g = item % groups;
      const int x0 = bin_start(px, grid_w, pool_w), x1 = bin_end(px, grid_w, pool_w);
      for (int y = y0 + ys; y < y1; y += ysplit) {
        const T* row = qs + ((long long)y * grid_w + x0) * d + g * 8;
        const int w = x1 - x0;
        int x = 0;
        for (; x + 8 <= w; x += 8) {       // eight independent 16-byte loads in flight
          uint4 raw[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) raw[u] = load16(row + (long long)(x + u) * d);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float v[8];
            unpack8(raw[u], row + (long long)(x + u) * d, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += v[i];
          }
        }
        for (; x < w; ++x) {
          float v[8];
          load8(row + (long long)x * d, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += v[i];
        }
      }
    }
    if (ysplit > 1) {
#pragma unroll
      for (int i = 0; i < 8; ++i) red[threadIdx.x * 8 + i] = acc[i];
      __syncthreads();
      if (item >= 0 && ys == 0) {
        for (int s2 = 1; s2 < ysplit; ++s2) {
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += red[(threadIdx.x + s2 * items) * 8 + i];
        }
      }
      __syncthreads();
    }
    if (item >= 0 && ys == 0) {
      const int px = item / groups, g = item % groups;
      const int x0 = bin_start(px, grid_w, pool_w), x1 = bin_end(px, grid_w, pool_w);
      const float inv = 1.f / (float)((y1 - y0) * (x1 - x0));
      const long long off = (bh * n_agents + (long long)py * pool_w + px) * d + g * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float m = acc[i] * inv;
        if (a_f32) a_f32[off + i] = m;
        if (a_lowp) a_lowp[off + i] = from_f32<T>(m);
      }
    }
  }
}

// ------------------------------------------------- generic online attention
constexpr int kSimtRows = 64;    // rows per CTA
constexpr int kSimtCols = 32;    // columns per chunk (one per lane)
constexpr int kSimtThreads = 256;

struct SimtAttendArgs {
  const void* rows;          // row vectors (agents or queries)
  long long rows_bstride, rows_hstride;
  const void* cols;          // column vectors (keys or agents)
  long long cols_bstride, cols_hstride;
  const void* vals;          // values (V or V_A), same row count as cols
  long long vals_bstride, vals_hstride;
  int H, n_rows, n_cols, d;
  float scale_log2;          // scale * log2(e)
  int row_blocks;
  int splits, cols_per_split;
  // partial output (splits > 0 && part_u != nullptr): unnormalised U, running
  // max m (log2 units) and sum l per row, slot = split index.
  float* part_u;             // [BH][slots][n_rows][d]
  float* part_ml;            // [BH][slots][n_rows][2]
  int slots;
  // normalised output (part_u == nullptr): out[bh][row][c] = U / l
  void* out;
  long long out_bstride, out_hstride;
};

__host__ __forceinline__ size_t simt_attend_smem_bytes(int d) {
  return sizeof(float) * ((size_t)kSimtRows * (d + 1) + (size_t)kSimtCols * (d + 1) +
                          (size_t)kSimtCols * d + (size_t)kSimtRows * (kSimtCols + 1) +
                          (size_t)kSimtRows * d + 3 * kSimtRows);
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) simt_attend_kernel(SimtAttendArgs p) {
  extern __shared__ float smem[];
  const int d = p.d, dp = d + 1;
  float* s_rows = smem;                                  // [R][d+1]
  float* s_cols = s_rows + kSimtRows * dp;               // [C][d+1]
  float* s_vals = s_cols + kSimtCols * dp;               // [C][d]
  float* s_p = s_vals + kSimtCols * d;                   // [R][C+1]
  float* s_u = s_p + kSimtRows * (kSimtCols + 1);        // [R][d]
  float* s_m = s_u + kSimtRows * d;
  float* s_l = s_m + kSimtRows;
  float* s_alpha = s_l + kSimtRows;

  long long idx = blockIdx.x;
  const int rb = (int)(idx % p.row_blocks);
  idx /= p.row_blocks;
  const int split = (int)(idx % p.splits);
  const long long bh = idx / p.splits;
  const int r0 = rb * kSimtRows;
  const int c_begin = split * p.cols_per_split;
  int c_end = c_begin + p.cols_per_split;
  if (c_end > p.n_cols) c_end = p.n_cols;

  const T* rows = static_cast<const T*>(p.rows) +
                  agent_set_offset(bh, p.H, p.rows_bstride, p.rows_hstride);
  const T* cols = static_cast<const T*>(p.cols) +
                  agent_set_offset(bh, p.H, p.cols_bstride, p.cols_hstride);
  const T* vals = static_cast<const T*>(p.vals) +
                  agent_set_offset(bh, p.H, p.vals_bstride, p.vals_hstride);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int e = tid; e < kSimtRows * d; e += kSimtThreads) {
    const int r = e / d, c = e % d;
    s_rows[r * dp + c] = (r0 + r < p.n_rows) ? to_f32(rows[(long long)(r0 + r) * d + c]) : 0.f;
    s_u[e] = 0.f;
  }
  for (int r = tid; r < kSimtRows; r += kSimtThreads) {
    s_m[r] = -INFINITY;
    s_l[r] = 0.f;
  }
  __syncthreads();

  for (int c0 = c_begin; c0 < c_end; c0 += kSimtCols) {
    const int valid = min(kSimtCols, c_end - c0);
    for (int e = tid; e < kSimtCols * d; e += kSimtThreads) {
      const int j = e / d, c = e % d;
      const bool ok = j < valid;
      s_cols[j * dp + c] = ok ? to_f32(cols[(long long)(c0 + j) * d + c]) : 0.f;
      s_vals[e] = ok ? to_f32(vals[(long long)(c0 + j) * d + c]) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < kSimtRows * kSimtCols; e += kSimtThreads) {
      const int r = e / kSimtCols, j = e % kSimtCols;
      const float* a = s_rows + r * dp;
      const float* b = s_cols + j * dp;
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(a[c], b[c], acc);
      s_p[r * (kSimtCols + 1) + j] = acc * p.scale_log2;
    }
    __syncthreads();
    for (int r = warp; r < kSimtRows; r += kSimtThreads / 32) {
      const bool ok = lane < valid;
      const float s = ok ? s_p[r * (kSimtCols + 1) + lane] : -INFINITY;
      float mx = s;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = s_m[r];
      const float m_new = fmaxf(m_old, mx);
      const float pr = ok ? exp2f(s - m_new) : 0.f;
      float sum = pr;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      s_p[r * (kSimtCols + 1) + lane] = pr;
      __syncwarp();
      if (lane == 0) {
        const float alpha = exp2f(m_old - m_new);   // 0 on the first chunk (m_old = -inf)
        s_alpha[r] = alpha;
        s_l[r] = s_l[r] * alpha + sum;
        s_m[r] = m_new;
      }
    }
    __syncthreads();
    for (int e = tid; e < kSimtRows * d; e += kSimtThreads) {
      const int r = e / d, c = e % d;
      const float* pr = s_p + r * (kSimtCols + 1);
      float acc = s_u[e] * s_alpha[r];
      for (int j = 0; j < valid; ++j) acc = fmaf(pr[j], s_vals[j * d + c], acc);
      s_u[e] = acc;
    }
    __syncthreads();
  }

  if (p.part_u != nullptr) {
    const long long slot_base = (bh * p.slots + split) * (long long)p.n_rows;
    for (int e = tid; e < kSimtRows * d; e += kSimtThreads) {
      const int r = e / d, c = e % d;
      if (r0 + r < p.n_rows) p.part_u[(slot_base + r0 + r) * d + c] = s_u[e];
    }
    for (int r = tid; r < kSimtRows; r += kSimtThreads) {
      if (r0 + r < p.n_rows) {
        p.part_ml[(slot_base + r0 + r) * 2 + 0] = s_m[r];
        p.part_ml[(slot_base + r0 + r) * 2 + 1] = s_l[r];
      }
    }
  } else {
    T* out = static_cast<T*>(p.out) + agent_set_offset(bh, p.H, p.out_bstride, p.out_hstride);
    for (int e = tid; e < kSimtRows * d; e += kSimtThreads) {
      const int r = e / d, c = e % d;
      if (r0 + r < p.n_rows) out[(long long)(r0 + r) * d + c] = from_f32<T>(s_u[e] / s_l[r]);
    }
  }
}

// ------------------------------------------------------------------ merge
// One warp per (slice, agent row): V_A = sum_s 2^(m_s - M) U_s / sum_s 2^(m_s - M) l_s.
// Lane s owns split s's weight (computed once); the weights are broadcast by
// shuffles while the lanes sweep the d columns of every split's partial row.
template <typename T>
__global__ void __launch_bounds__(256) agent_merge_kernel(const float* __restrict__ part_u,
                                                          const float* __restrict__ part_ml,
                                                          SplitPlan plan, long long BH,
                                                          int n_agents, int d,
                                                          float* __restrict__ va_f32,
                                                          T* __restrict__ va_lowp) {
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= BH * n_agents) return;
  const long long bh = row / n_agents;
  const int j = (int)(row % n_agents);
  const int n_splits = splits_of_slice(plan, bh);
  const long long slot0 = bh * plan.slots;
  float mx = -INFINITY;
  for (int s = lane; s < n_splits; s += 32)
    mx = fmaxf(mx, part_ml[((slot0 + s) * n_agents + j) * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f, den = 0.f;
  for (int s0 = 0; s0 < n_splits; s0 += 32) {
    float w = 0.f;
    if (s0 + lane < n_splits) {
      const float* ml = part_ml + ((slot0 + s0 + lane) * n_agents + j) * 2;
      w = exp2f(ml[0] - mx);
      den += w * ml[1];
    }
    const int cnt = min(32, n_splits - s0);
    const long long stride = (long long)n_agents * d;      // between consecutive splits
    const float* base = part_u + ((slot0 + s0) * n_agents + j) * (long long)d;
    for (int s = 0; s < cnt; s += 4) {                      // four splits' loads in flight
      float u[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = lane + 32 * q;
          u[a][q] = (s + a < cnt && c < d) ? base[(s + a) * stride + c] : 0.f;
        }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float ws = __shfl_sync(0xffffffffu, w, (s + a) & 31);
        const float wa = (s + a < cnt) ? ws : 0.f;
        acc0 = fmaf(wa, u[a][0], acc0);
        acc1 = fmaf(wa, u[a][1], acc1);
        acc2 = fmaf(wa, u[a][2], acc2);
        acc3 = fmaf(wa, u[a][3], acc3);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  const float inv = 1.f / den;
  const float accs[4] = {acc0, acc1, acc2, acc3};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = lane + 32 * q;
    if (c < d) {
      const float v = accs[q] * inv;
      const long long o = row * d + c;
      if (va_f32) va_f32[o] = v;
      if (va_lowp) va_lowp[o] = from_f32<T>(v);
    }
  }
}

}  // namespace aa
