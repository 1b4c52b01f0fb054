// Depth-wise 3x3 convolution of V over the token grid, added to the attention
// output: the DWC term of the full Agent Attention module (the arXiv
// 2312.08874v3 summary, §4 "Module Enhancements": a depth-wise convolution
// term of cost k^2 N C with k = 3).
//
// Each thread owns a run of kDwcSpan neighbouring tokens of one grid row and
// one 8-channel group of a (batch, head) slice: it reads the 3 x (kDwcSpan+2)
// neighbouring 8-channel groups of V once (zero outside the grid), applies the
// head's per-channel 3x3 kernels (staged in shared memory as [tap][channel],
// each weight vector read once for the whole run), adds the bias and, when
// accumulating, the value already in `out`, and writes the run.  Consecutive
// threads cover consecutive channel groups of consecutive runs, so every tap
// row is a coalesced read and blocks share rows through L1/L2.  HBM-bound:
// V read once, out read (when accumulating) and written once.
#pragma once

#include "common.cuh"

namespace aa {

constexpr int kDwcThreads = 256;

__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 raw;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = raw;
}

// Tokens per thread along x: neighbouring outputs share 2 of their 3 tap
// columns and every weight vector.
constexpr int kDwcSpan = 2;

// v, out: [BH][grid_h*grid_w][d] of T; w: [H][d][3][3] fp32; bias: [H][d] fp32
// or null.  Thread = (grid row y, run of kDwcSpan tokens along x, 8-channel
// group); grid: (ceil(items / kDwcThreads), min(BH, 65535)) with
// items = grid_h * ceil(grid_w / kDwcSpan) * d/8 < 2^31.  With programmatic
// dependent launch the convolution is computed before waiting for the
// previous kernel of the stream (which writes `out`, not V).
template <typename T>
__global__ void __launch_bounds__(kDwcThreads)
    dwc_kernel(const T* __restrict__ v, const float* __restrict__ w,
               const float* __restrict__ bias, T* __restrict__ out, int H, int grid_h,
               int grid_w, int d, long long BH, int accumulate) {
  extern __shared__ float s_w[];   // [9][d] kernel taps, then [d] bias
  pdl_trigger();
  const unsigned nch = (unsigned)d / 8u;
  const unsigned xruns = ((unsigned)grid_w + kDwcSpan - 1) / kDwcSpan;
  const unsigned N = (unsigned)grid_h * (unsigned)grid_w;
  const unsigned items = (unsigned)grid_h * xruns * nch;
  const unsigned item = blockIdx.x * blockDim.x + threadIdx.x;
  const bool mine = item < items;
  const unsigned ch = mine ? item % nch : 0u;
  const unsigned run = mine ? item / nch : 0u;
  const int y = (int)(run / xruns);
  const int x0 = (int)(run - (unsigned)y * xruns) * kDwcSpan;
  for (long long bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const int h = (int)(bh % H);
    __syncthreads();   // the previous slice's weights are no longer read
    for (int i = threadIdx.x; i < 9 * d; i += blockDim.x) {
      const int tap = i / d, c = i - tap * d;
      s_w[i] = w[((long long)h * d + c) * 9 + tap];
    }
    for (int i = threadIdx.x; i < d; i += blockDim.x) s_w[9 * d + i] = bias ? bias[h * d + i] : 0.f;
    __syncthreads();
    float acc[kDwcSpan][8];
    const T* vs = v + bh * (long long)N * d + ch * 8;
    if (mine) {
#pragma unroll
      for (int t = 0; t < kDwcSpan; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[t][e] = s_w[9 * d + ch * 8 + e];
#pragma unroll
      for (int ty = 0; ty < 3; ++ty) {
        const int yy = y + ty - 1;
        if (yy < 0 || yy >= grid_h) continue;
        // the kDwcSpan + 2 tap columns x0-1 .. x0+kDwcSpan of row yy, kept as
        // raw 16-byte rows and widened at each use (fewer live registers)
        uint4 raw[kDwcSpan + 2];
        const T* cp[kDwcSpan + 2];
        bool cin[kDwcSpan + 2];
#pragma unroll
        for (int c = 0; c < kDwcSpan + 2; ++c) {
          const int xx = x0 + c - 1;
          cin[c] = xx >= 0 && xx < grid_w;
          cp[c] = vs + (size_t)((unsigned)yy * grid_w + (cin[c] ? xx : 0)) * d;
          raw[c] = cin[c] ? load16(cp[c]) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int tx = 0; tx < 3; ++tx) {
          float wt[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) wt[e] = s_w[(ty * 3 + tx) * d + ch * 8 + e];
#pragma unroll
          for (int t = 0; t < kDwcSpan; ++t) {
            if (!cin[t + tx]) continue;
            float cv[8];
            unpack8(raw[t + tx], cp[t + tx], cv);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[t][e] = fmaf(wt[e], cv[e], acc[t][e]);
          }
        }
      }
    }
    pdl_wait();   // `out` may be written by the previous kernel of the stream
    if (mine) {
#pragma unroll
      for (int t = 0; t < kDwcSpan; ++t) {
        if (x0 + t >= grid_w) continue;
        T* o = out + (bh * (long long)N + (long long)y * grid_w + x0 + t) * d + ch * 8;
        if (accumulate) {
          float prev[8];
          load8(o, prev);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[t][e] += prev[e];
        }
        store8(o, acc[t]);
      }
    }
  }
}

}  // namespace aa
