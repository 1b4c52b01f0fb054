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
// The host uses this kernel when the tile of one agent column fits the
// shared-memory budget and falls back to agent_pool_kernel otherwise.
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

}  // namespace aa
