// Device helpers shared by the Agent Attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace aa {

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream runs; it
// must wait here before touching anything that kernel writes (a no-op when
// the kernel was launched normally).  The trigger lets the next kernel of the
// stream begin its own launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr float kLog2e = 1.4426950408889634f;

// Element loads/stores for the two run dtypes, widened to / narrowed from fp32.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load 8 consecutive elements (16-byte aligned for bf16, 32 for fp32) as fp32.
__device__ __forceinline__ void load8(const float* p, float (&out)[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&out)[8]) {
  uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}

// Raw 16-byte load and its widening (8 bf16 or, for fp32, the first of two
// halves: fp32 rows are read as two 16-byte halves by the caller's unpack).
__device__ __forceinline__ uint4 load16(const __nv_bfloat16* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ uint4 load16(const float* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ void unpack8(const uint4& raw, const __nv_bfloat16*, float (&out)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
// fp32: 8 values span 32 bytes; `raw` holds the first 16, the rest is reloaded.
__device__ __forceinline__ void unpack8(const uint4& raw, const float* p, float (&out)[8]) {
  out[0] = __uint_as_float(raw.x);
  out[1] = __uint_as_float(raw.y);
  out[2] = __uint_as_float(raw.z);
  out[3] = __uint_as_float(raw.w);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

// Adaptive pooling bin [start, end) of bin i when an axis of length g is cut
// into p bins: [floor(i*g/p), ceil((i+1)*g/p)).
__host__ __device__ __forceinline__ int bin_start(int i, int g, int p) {
  return (int)(((long long)i * g) / p);
}
__host__ __device__ __forceinline__ int bin_end(int i, int g, int p) {
  return (int)((((long long)i + 1) * g + p - 1) / p);
}

// Element offset of the agent set of slice bh (b = bh / H, h = bh % H).
__host__ __device__ __forceinline__ long long agent_set_offset(long long bh, int H,
                                                               long long batch_stride,
                                                               long long head_stride) {
  return (bh / H) * batch_stride + (bh % H) * head_stride;
}

// Split-over-keys bookkeeping shared by the aggregation kernels and the merge.
// Two schedules exist:
//  * fixed: every slice has `fixed` splits of `cols_per_split` keys;
//  * stream: `ctas` CTAs cut the slices' key tiles (tiles_per_slice tiles of
//    `tile` keys per slice, total_tiles over all slices) into contiguous,
//    equal-as-possible ranges; CTA c owns global tiles
//    [floor(c*total/ctas), floor((c+1)*total/ctas)) and writes one partial
//    per slice its range touches, in slot (c - first CTA of that slice).
struct SplitPlan {
  int fixed;                 // > 0: fixed schedule
  int ctas;                  // stream schedule
  long long total_tiles;
  int tiles_per_slice;
  int slots;                 // partial slots reserved per slice
};

__host__ __device__ __forceinline__ long long stream_tile_begin(const SplitPlan& p, long long c) {
  return (c * p.total_tiles) / p.ctas;
}
// First CTA whose range contains global tile t.
__host__ __device__ __forceinline__ long long stream_cta_of_tile(const SplitPlan& p, long long t) {
  return ((t + 1) * p.ctas - 1) / p.total_tiles;
}
__host__ __device__ __forceinline__ int splits_of_slice(const SplitPlan& p, long long bh) {
  if (p.fixed > 0) return p.fixed;
  long long t0 = bh * p.tiles_per_slice;
  long long t1 = t0 + p.tiles_per_slice - 1;
  return (int)(stream_cta_of_tile(p, t1) - stream_cta_of_tile(p, t0) + 1);
}

// Launches `kernel`; with pdl = true, with programmatic stream serialization
// (the kernel may start before the previous kernel of the stream finishes and
// synchronises with it through pdl_wait()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t st, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace aa
