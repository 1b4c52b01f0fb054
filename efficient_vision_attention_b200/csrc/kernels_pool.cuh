// Agent pooling with the bin rows staged in shared memory by bulk async copies.
//
// One CTA per (slice, agent row py, chunk of agent columns): thread 0 issues
// one cp.async.bulk per grid row of the bin (the row segment of the chunk's
// token columns is contiguous in memory) onto one mbarrier, so a CTA keeps its
// whole tile in flight without holding it in registers, and several CTAs per
// SM overlap their loads.  Then phase 1 sums every token column of the tile
// over the bin's rows (threads over (column, 8-channel group), conflict-free
// 16-byte shared loads) and phase 2 adds the columns of each agent's bin and
// divides by its token count.  fp32 sums.  Bins follow the adaptive-pool
// convention [floor(iG/P), ceil((i+1)G/P)) (they may overlap by one token).
// The host sends bf16 Q with bins of at most 64 rows (grid sides up to 46340)
// to agent_pool_band_kernel below; otherwise it uses this kernel when the
// tile of one agent column fits the shared-memory budget, else
// agent_pool_kernel.
#pragma once

#include "common.cuh"
#include "tc_primitives.cuh"

namespace aa {

constexpr int kPoolTmaThreads = 256;
constexpr int kPoolTmaTileBudget = 56 * 1024;   // bytes of staged Q per CTA

struct PoolTmaPlan {
  int px_per_cta;
  int rows_max;      // tallest bin
  int cols_max;      // widest chunk of token columns
  size_t smem;
  bool ok;
};

inline PoolTmaPlan pool_tma_plan(int grid_h, int grid_w, int pool_h, int pool_w, int d,
                                 int elem) {
  PoolTmaPlan pl{0, 0, 0, 0, false};
  for (int py = 0; py < pool_h; ++py) {
    const int h = bin_end(py, grid_h, pool_h) - bin_start(py, grid_h, pool_h);
    if (h > pl.rows_max) pl.rows_max = h;
  }
  const int groups = d / 8;
  // fewest chunks of equal agent-column count whose tile fits the budget
  for (int n = 1; n <= pool_w; ++n) {
    const int per = (pool_w + n - 1) / n;
    int cols = 0;
    for (int px0 = 0; px0 < pool_w; px0 += per) {
      const int px1 = px0 + per < pool_w ? px0 + per : pool_w;
      const int c = bin_end(px1 - 1, grid_w, pool_w) - bin_start(px0, grid_w, pool_w);
      if (c > cols) cols = c;
    }
    const size_t tile = (size_t)pl.rows_max * cols * d * elem;
    if (tile <= (size_t)kPoolTmaTileBudget && per * groups <= kPoolTmaThreads) {
      pl.px_per_cta = per;
      pl.cols_max = cols;
      pl.smem = 128 + ((tile + 127) & ~(size_t)127) + (size_t)cols * d * sizeof(float) + 16;
      pl.ok = true;
      return pl;
    }
  }
  return pl;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}

// Shared memory: [tile region: rows x cols x d of T, tile_region bytes]
// [column sums: cols_max x d floats][mbarrier].
template <typename T>
__global__ void __launch_bounds__(kPoolTmaThreads) agent_pool_tma_kernel(
    const T* __restrict__ q, float* __restrict__ a_f32, T* __restrict__ a_lowp, int N, int d,
    int grid_h, int grid_w, int pool_h, int pool_w, int px_per_cta, int cols_max,
    int tile_region) {
  extern __shared__ uint8_t pool_smem[];
  pdl_trigger();
  // 128-byte aligned by pointer arithmetic on the shared array, so the
  // compiler keeps the shared address space for every access through it
  uint8_t* base = pool_smem + ((128u - (tc::smem_u32(pool_smem) & 127u)) & 127u);
  T* tile = reinterpret_cast<T*>(base);
  float* colsum = reinterpret_cast<float*>(base + tile_region);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + tile_region + (size_t)cols_max * d * 4);

  const int n_chunks = (pool_w + px_per_cta - 1) / px_per_cta;
  const int py = blockIdx.x / n_chunks;
  const int px0 = (blockIdx.x % n_chunks) * px_per_cta;
  const int px1 = min(pool_w, px0 + px_per_cta);
  const long long bh = blockIdx.y;
  const int y0 = bin_start(py, grid_h, pool_h), y1 = bin_end(py, grid_h, pool_h);
  const int xs = bin_start(px0, grid_w, pool_w), xe = bin_end(px1 - 1, grid_w, pool_w);
  const int rows = y1 - y0, cols = xe - xs, groups = d >> 3;
  const uint32_t row_bytes = (uint32_t)((size_t)cols * d * sizeof(T));

  if (threadIdx.x == 0) {
    tc::mbar_init(bar, 1);
    tc::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    tc::mbar_expect_tx(bar, (uint32_t)rows * row_bytes);
    const T* src = q + (bh * (long long)N + (long long)y0 * grid_w + xs) * d;
    for (int r = 0; r < rows; ++r)
      bulk_load(reinterpret_cast<uint8_t*>(tile) + (size_t)r * row_bytes,
                src + (long long)r * grid_w * d, row_bytes, bar);
  }
  // bounded wait for the tile; on expiry the CTA writes nothing and raises
  // the watchdog (the copies are then waited for once more before exit)
  bool ok = true;
  {
    const uint64_t t0 = tc::globaltimer();
    while (!tc::mbar_try_wait(bar, 0)) {
      if (tc::globaltimer() - t0 > tc::kWaitLimitNs) {
        ok = false;
        atomicOr(&tc::g_watchdog, 1u);
        break;
      }
    }
  }
  ok = __syncthreads_and(ok) != 0;    // every thread takes the same path
  if (!ok) {
    const uint64_t t0 = tc::globaltimer();
    while (!tc::mbar_try_wait(bar, 0) && tc::globaltimer() - t0 < tc::kWaitLimitNs) {
    }
    return;
  }
  // phase 1: column sums over the bin's rows
  for (int it = threadIdx.x; it < cols * groups; it += blockDim.x) {
    const int x = it / groups, g = it - x * groups;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    const T* cp = tile + (size_t)x * d + g * 8;
    for (int r = 0; r < rows; ++r) {
      float v[8];
      load8(cp + (size_t)r * cols * d, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += v[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) colsum[(size_t)it * 8 + i] = acc[i];
  }
  __syncthreads();
  // phase 2: bin sums over the columns of each agent of the chunk
  const long long n_agents = (long long)pool_h * pool_w;
  for (int it = threadIdx.x; it < (px1 - px0) * groups; it += blockDim.x) {
    const int px = px0 + it / groups, g = it % groups;
    const int bx0 = bin_start(px, grid_w, pool_w), bx1 = bin_end(px, grid_w, pool_w);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int x = bx0; x < bx1; ++x) {
      const float* cs = colsum + ((size_t)(x - xs) * groups + g) * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += cs[i];
    }
    const float inv = 1.f / (float)(rows * (bx1 - bx0));
    const long long off = (bh * n_agents + (long long)py * pool_w + px) * d + g * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float m = acc[i] * inv;
      if (a_f32) a_f32[off + i] = m;
      if (a_lowp) a_lowp[off + i] = from_f32<T>(m);
    }
  }
}


// ------------------------------------------------ bins of at most 64 rows, bf16 Q
// A CTA takes the grid rows [y0, y1) of one agent row py (the bin rows, 64 at
// most) and the token columns of a chunk of consecutive agent columns of one
// slice: a thread per (token column, 8-channel group) issues the loads of its
// column kBatch rows at a time (in flight together, straight into registers,
// no staging), sums them in fp32 into a shared column sum, and a thread per
// (agent, 8-channel group) then adds the columns [x0, x1) of its bin and
// divides by its token count.  Adaptive bins [floor(iG/P), ceil((i+1)G/P))
// may overlap by one token: a column shared by two bins of the chunk is
// summed once and used by both.  kBatch is 4 for bins of up to 4 rows, else
// 8 (taller bins loop over 8-row batches): the batch's registers bound how
// many CTAs share an SM, and with 16 rows' loads in flight a thread needed
// about 108 registers (3 CTAs of 160 threads per SM, 2.3 waves on the
// SD-latent grid) against 56 for 8 rows (7 CTAs, one wave).
constexpr int kPoolBandBatch = 8;       // largest batch of a column's loads in flight together
constexpr int kPoolBandMaxRows = 64;
constexpr int kPoolBandMaxSide = 46340;   // grid sides whose bin products fit 32 bits
inline int pool_band_batch(int rows) { return rows <= 4 ? 4 : kPoolBandBatch; }
// The adaptive bin bounds in 32-bit arithmetic (exact for sides <= 46340:
// (i + 1) g + p - 1 <= g^2 + g < 2^31).
__device__ __forceinline__ int band_bin_start(int i, int g, int p) { return (i * g) / p; }
__device__ __forceinline__ int band_bin_end(int i, int g, int p) { return ((i + 1) * g + p - 1) / p; }

struct PoolBandPlan {
  int rows_max;      // tallest bin
  int bins;          // agent columns per chunk (a divisor of pool_w, or pool_w)
  int threads;
  size_t smem;
  bool ok;
};

inline PoolBandPlan pool_band_plan(int grid_h, int grid_w, int pool_h, int pool_w, int d) {
  PoolBandPlan pl{0, 0, 0, 0, false};
  if (d % 8 != 0 || pool_h < 1 || pool_w < 1 || pool_h > grid_h || pool_w > grid_w ||
      grid_h > kPoolBandMaxSide || grid_w > kPoolBandMaxSide)
    return pl;
  for (int py = 0; py < pool_h; ++py) {
    const int h = bin_end(py, grid_h, pool_h) - bin_start(py, grid_h, pool_h);
    if (h > pl.rows_max) pl.rows_max = h;
  }
  if (pl.rows_max > kPoolBandMaxRows) return pl;
  const int groups = d / 8;
  // whole bins per chunk: the fewest that divide pool_w and span at least
  // 32 token columns (all of them when no smaller divisor does)
  const int min_w = grid_w / pool_w;                 // narrowest bin, >= 1
  const int want = (32 + min_w - 1) / min_w;
  pl.bins = pool_w;
  for (int b = 1; b < pool_w; ++b)
    if (pool_w % b == 0 && b >= want) {
      pl.bins = b;
      break;
    }
  int cols_max = 0;
  for (int px0 = 0; px0 < pool_w; px0 += pl.bins) {
    const int c = bin_end(px0 + pl.bins - 1, grid_w, pool_w) - bin_start(px0, grid_w, pool_w);
    if (c > cols_max) cols_max = c;
  }
  const int items = cols_max * groups;
  pl.threads = ((items + 31) / 32) * 32;
  if (pl.threads > 1024) return pl;
  pl.smem = (size_t)items * 8 * sizeof(float);
  pl.ok = pl.smem <= 48 * 1024;
  return pl;
}

template <typename T, int kBatch>
__global__ void __maxnreg__(kBatch <= 4 ? 48 : 64)
    agent_pool_band_kernel(const __nv_bfloat16* __restrict__ q,
                                       float* __restrict__ a_f32, T* __restrict__ a_lowp, int N,
                                       int d, int grid_h, int grid_w, int pool_h, int pool_w,
                                       int bins) {
  extern __shared__ float band_colsum[];
  pdl_trigger();
  const int n_chunks = pool_w / bins;
  const int py = blockIdx.x / n_chunks, ch = blockIdx.x - py * n_chunks;
  const long long bh = blockIdx.y;
  const int groups = d >> 3;
  const int y0 = band_bin_start(py, grid_h, pool_h);
  const int rows = band_bin_end(py, grid_h, pool_h) - y0;
  const int px0 = ch * bins;
  const int xs = band_bin_start(px0, grid_w, pool_w);
  const int items = (band_bin_end(px0 + bins - 1, grid_w, pool_w) - xs) * groups;
  const int it = threadIdx.x;
  if (it < items) {
    const int x = it / groups, g = it - x * groups;
    const __nv_bfloat16* src =
        q + (bh * (long long)N + (long long)y0 * grid_w + xs + x) * d + g * 8;
    const long long row_step = (long long)grid_w * d;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    // 32-bit offsets in 16-byte units from one base address: a band spans
    // at most 64 x 46340 x 128 elements / 8 < 2^32 such units
    const uint4* base = reinterpret_cast<const uint4*>(src);
    const uint32_t step = (uint32_t)(row_step >> 3);
    if (rows <= kBatch) {
      // bins of up to kBatch rows: every load of the column in flight at once
      uint4 raw[kBatch];
#pragma unroll
      for (int r = 0; r < kBatch; ++r)
        if (r < rows) raw[r] = __ldcs(base + r * step);
#pragma unroll
      for (int r = 0; r < kBatch; ++r) {
        if (r < rows) {
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[r]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            acc[2 * i] += f.x;
            acc[2 * i + 1] += f.y;
          }
        }
      }
    } else {
      // taller bins: kBatch rows' loads in flight at a time
      for (int rb = 0; rb < rows; rb += kBatch) {
        uint4 raw[kBatch];
#pragma unroll
        for (int r = 0; r < kBatch; ++r)
          if (rb + r < rows) raw[r] = __ldcs(base + (uint32_t)(rb + r) * step);
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
          if (rb + r < rows) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[r]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __bfloat1622float2(h[i]);
              acc[2 * i] += f.x;
              acc[2 * i + 1] += f.y;
            }
          }
        }
      }
    }
    float4* cs = reinterpret_cast<float4*>(band_colsum + (size_t)it * 8);
    cs[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    cs[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  __syncthreads();
  if (it < bins * groups) {
    const int pxl = it / groups, g = it - pxl * groups;
    const int px = px0 + pxl;
    const int x0 = band_bin_start(px, grid_w, pool_w) - xs;
    const int x1 = band_bin_end(px, grid_w, pool_w) - xs;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int x = x0; x < x1; ++x) {
      const float4* cs = reinterpret_cast<const float4*>(band_colsum + ((size_t)x * groups + g) * 8);
      const float4 a = cs[0], b = cs[1];
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    const float inv = 1.f / (float)(rows * (x1 - x0));
    const long long off = (bh * pool_h * (long long)pool_w + (long long)py * pool_w + px) * d + g * 8;
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = acc[i] * inv;
    if (a_f32) {
      *reinterpret_cast<float4*>(a_f32 + off) = make_float4(m[0], m[1], m[2], m[3]);
      *reinterpret_cast<float4*>(a_f32 + off + 4) = make_float4(m[4], m[5], m[6], m[7]);
    }
    if (a_lowp) {
#pragma unroll
      for (int i = 0; i < 8; ++i) a_lowp[off + i] = from_f32<T>(m[i]);
    }
  }
}

}  // namespace aa
