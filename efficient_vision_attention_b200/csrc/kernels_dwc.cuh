// Depth-wise 3x3 convolution of V over the token grid, added to the attention
// output: the DWC term of the full Agent Attention module (the arXiv
// 2312.08874v3 summary, §4 "Module Enhancements": a depth-wise convolution
// term of cost k^2 N C with k = 3).
//
// Each thread owns one (token, 8-channel group) of one (batch, head) slice:
// it reads the 9 neighbouring 8-channel groups of V (zero outside the grid),
// applies the head's per-channel 3x3 kernels (staged in shared memory as
// [tap][channel]), adds the bias and, when accumulating, the value already in
// `out`, and writes 8 channels.  Consecutive threads cover consecutive
// channel groups of consecutive tokens, so every tap is a coalesced row read
// and the 9 taps of a block hit L1/L2 for the rows they share.  HBM-bound:
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

// The 9 taps of one (token, 8-channel group): raw 16-byte bf16 rows (zero
// outside the grid), loaded before anything else so that their trip to
// memory overlaps the staging of the kernel weights.
struct DwcTaps {
  uint4 raw[9];
};
__device__ __forceinline__ void dwc_load_taps(const __nv_bfloat16* vs, int y, int x, int grid_h,
                                              int grid_w, int d, DwcTaps& t) {
#pragma unroll
  for (int ty = 0; ty < 3; ++ty) {
#pragma unroll
    for (int tx = 0; tx < 3; ++tx) {
      const int yy = y + ty - 1, xx = x + tx - 1;
      const bool in = yy >= 0 && yy < grid_h && xx >= 0 && xx < grid_w;
      t.raw[ty * 3 + tx] =
          in ? __ldg(reinterpret_cast<const uint4*>(vs + (size_t)((unsigned)yy * grid_w + xx) * d))
             : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// v, out: [BH][grid_h*grid_w][d] of T; w: [H][d][3][3] fp32; bias: [H][d] fp32
// or null.  Grid: (ceil(N*d/8 / kDwcThreads), min(BH, 65535)), N*d/8 < 2^31.
// With programmatic dependent launch the V taps are read and convolved before
// waiting for the previous kernel of the stream (which writes `out`, not V).
template <typename T>
__global__ void __launch_bounds__(kDwcThreads)
    dwc_kernel(const T* __restrict__ v, const float* __restrict__ w,
               const float* __restrict__ bias, T* __restrict__ out, int H, int grid_h,
               int grid_w, int d, long long BH, int accumulate) {
  extern __shared__ float s_w[];   // [9][d] kernel taps, then [d] bias
  pdl_trigger();
  const unsigned nch = (unsigned)d / 8u;
  const unsigned N = (unsigned)grid_h * (unsigned)grid_w;
  const unsigned item = blockIdx.x * blockDim.x + threadIdx.x;
  const bool mine = item < N * nch;
  const unsigned n = mine ? item / nch : 0u;
  const unsigned ch = item - n * nch;
  const int y = (int)(n / (unsigned)grid_w), x = (int)(n - (unsigned)y * grid_w);
  for (long long bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const int h = (int)(bh % H);
    const T* vs = v + bh * (long long)N * d + ch * 8;
    DwcTaps taps;
    constexpr bool kPreload = false;   // preloading the 9 taps (93 registers) measured slower
    if constexpr (kPreload) {
      if (mine) dwc_load_taps(vs, y, x, grid_h, grid_w, d, taps);
    }
    __syncthreads();   // the previous slice's weights are no longer read
    for (int i = threadIdx.x; i < 9 * d; i += blockDim.x) {
      const int tap = i / d, c = i - tap * d;
      s_w[i] = w[((long long)h * d + c) * 9 + tap];
    }
    for (int i = threadIdx.x; i < d; i += blockDim.x) s_w[9 * d + i] = bias ? bias[h * d + i] : 0.f;
    __syncthreads();
    float acc[8];
    if (mine) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = s_w[9 * d + ch * 8 + e];
#pragma unroll
      for (int tap = 0; tap < 9; ++tap) {
        float t[8];
        if constexpr (kPreload) {
          unpack8(taps.raw[tap], reinterpret_cast<const __nv_bfloat16*>(vs), t);
        } else {
          const int yy = y + tap / 3 - 1, xx = x + tap % 3 - 1;
          if (yy < 0 || yy >= grid_h || xx < 0 || xx >= grid_w) continue;
          load8(vs + (size_t)((unsigned)yy * grid_w + xx) * d, t);
        }
        const float* wt = s_w + tap * d + ch * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wt[e], t[e], acc[e]);
      }
    }
    pdl_wait();   // `out` may be written by the previous kernel of the stream
    if (mine) {
      T* o = out + (bh * (long long)N + n) * d + ch * 8;
      if (accumulate) {
        float prev[8];
        load8(o, prev);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += prev[e];
      }
      store8(o, acc);
    }
  }
}

}  // namespace aa
