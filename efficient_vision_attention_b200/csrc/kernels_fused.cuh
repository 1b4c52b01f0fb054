// Whole forward pass of one small slice in one CTA (bf16, N <= 256 tokens,
// k <= 128 pooled or given agents, d <= 64): agent_fused_small_tc.
//
// For slices this small the four-kernel path is bound by its launches and
// hand-offs (a pool, a split aggregation whose partials go through HBM, a
// merge and a broadcast for a few hundred tokens).  Here one CTA per (b, h)
// stages Q, K and V once by TMA and runs every step on chip:
//
//   1. pool     A[a] = mean of Q over agent a's bin (adaptive bins), or the
//               given agent rows, written as bf16 in the 128-byte-swizzled
//               operand layout;
//   2. S1 = A K^T             tcgen05 SS, M = 128 agent rows, N = N rounded
//                              up to 16 (keys), into TMEM;
//   3. softmax over the keys, P1 as bf16 over its scores (two passes: row
//      maxima, then exponentials, with the row sums of slab_exp);
//   4. U = P1 V               tcgen05 TS (V as an MN-major operand);
//   5. V_A = U / l1 as bf16 in shared memory (MN-major operand layout);
//   6. S2 = Q A^T per 128-query tile, softmax over the agents, P2 over S2;
//   7. O = P2 V_A             tcgen05 TS, then 1/l2, bf16, staging, TMA store.
//
// 256 threads: 8 warps, two per TMEM lane quadrant, each owning a 16-row slab
// of the 128 TMEM lanes (the 16x256b access shape of the other tensor-core
// kernels, whose slab softmax routines this kernel reuses); thread 0 issues
// the TMA copies and the MMAs between phases.  TMEM: 256 columns, so two CTAs
// fit on an SM: S1 over [0, 256) with P1 over [0, 128); U over [128, 192)
// once S1 is read; then query tile t's S2 over [128 t, 128 t + kpad) with P2
// over its first 64 columns and O_t over [128 t + 64, 128 t + 64 + dn) once
// S2_t is read (kpad <= 128, dn <= 64).
// Every mbarrier wait is bounded; a CTA whose wait gives up skips the rest of
// its work (still meeting every __syncthreads) and raises the watchdog.
#pragma once

#include "common.cuh"
#include "kernels_tc.cuh"
#include "tc_primitives.cuh"

namespace aa {
namespace tc {

constexpr int kFusedThreads = 256;
constexpr int kFusedMaxN = 256;
constexpr int kFusedMaxAgents = 128;
constexpr int kFusedTmemCols = 256;

struct FusedBars {
  uint64_t tma_q;            // Q staged
  uint64_t tma_kv;           // K and V staged
  uint64_t mma;              // one phase per MMA batch (S1, P1 V, S2, P2 V_A)
  uint64_t chunk[4];         // arrivals of the slab softmax routines (never waited on)
  uint64_t drain;            // completion of every MMA before TMEM is released
  uint32_t tmem_base;
  int abort;
};

// Shared memory of a slice with rows_alloc = N rounded up to 16 token rows:
// Q | K | V (rows_alloc x 128 bytes each, 1024-byte aligned) | A (128 x 128)
// | barriers.  V_A goes over K (dead after S1), the O staging tiles over K
// and V (dead after step 4).  The second S2 tile may read Q rows up to 255,
// past Q's rows: those fall inside K's region and only feed output rows >= N.
struct FusedLayout {
  int rows_alloc, box_rows, n_box;
  uint32_t tensor_bytes;     // rows_alloc * 128
  size_t smem;
};

__host__ __device__ inline FusedLayout fused_layout(int N) {
  FusedLayout L;
  L.rows_alloc = round16(N);
  L.n_box = L.rows_alloc <= 128 ? 1 : 2;
  L.box_rows = L.rows_alloc / L.n_box;                 // a multiple of 8
  L.tensor_bytes = (uint32_t)L.rows_alloc * kRowBytes;
  // 1024 alignment slack + Q, K, V + A + barriers; K + V also hold V_A and
  // the two 16 KB O staging tiles.
  L.smem = 1024 + 3 * (size_t)L.tensor_bytes + (size_t)kFusedMaxAgents * kRowBytes +
           sizeof(FusedBars);
  return L;
}

__host__ __device__ inline bool fused_small_fits(int N, int d, int k) {
  if (N < 1 || N > kFusedMaxN || d < 8 || d > 64 || (d % 8) != 0 || k < 1 ||
      k > kFusedMaxAgents)
    return false;
  const FusedLayout L = fused_layout(N);
  // K + V must hold the O staging tiles (128 rows per 128-query tile)
  const int n_qt = (N + kQTile - 1) / kQTile;
  return 2 * (size_t)L.tensor_bytes >= (size_t)n_qt * kQTileBytes;
}


// Bounded wait without abort checks (the CTA is already giving up).
__device__ __forceinline__ void fused_drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kWaitLimitNs) {
  }
}

// Bounded wait of every thread of the CTA on a phase; all threads take the
// same outcome through the following __syncthreads_and.
__device__ __forceinline__ bool fused_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                           bool ok) {
  if (ok) ok = mbar_wait(bar, parity, abort);
  return __syncthreads_and(ok ? 1 : 0) != 0;
}

__global__ void __launch_bounds__(kFusedThreads, 2)
    agent_fused_small_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                                const __grid_constant__ CUtensorMap map_k,
                                const __grid_constant__ CUtensorMap map_v,
                                const __grid_constant__ CUtensorMap map_o, int N, int d,
                                int grid_h, int grid_w, int pool_h, int pool_w, int k, int H,
                                const __nv_bfloat16* __restrict__ agents, long long ag_bstride,
                                float c) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const FusedLayout L = fused_layout(N);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + L.tensor_bytes;
  uint8_t* sV = sK + L.tensor_bytes;
  uint8_t* sA = sV + L.tensor_bytes;
  uint8_t* sVA = sK;                                   // after S1
  uint8_t* sO = sK;                                    // after P1 V (two 16 KB tiles)
  FusedBars* bars = reinterpret_cast<FusedBars*>(sA + kFusedMaxAgents * kRowBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int kpad = round16(k);
  const int npad = L.rows_alloc;                       // keys, rounded up to 16
  const int d16 = (d + 15) >> 4;
  const int dn = d16 * 16;
  const int groups = d >> 3;                           // 8-channel groups of a row
  const int n_qt = (N + kQTile - 1) / kQTile;

  if (threadIdx.x == 0) {
    mbar_init(&bars->tma_q, 1);
    mbar_init(&bars->tma_kv, 1);
    mbar_init(&bars->mma, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&bars->chunk[i], kFusedThreads / 32);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    mbar_fence_init();
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_o);
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, kFusedTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (threadIdx.x == 0) {
    pdl_wait();
    // Q on its own barrier, so the pooling starts while K and V still load
    mbar_expect_tx(&bars->tma_q, (uint32_t)L.n_box * (uint32_t)L.box_rows * kRowBytes);
    mbar_expect_tx(&bars->tma_kv, 2u * (uint32_t)L.n_box * (uint32_t)L.box_rows * kRowBytes);
    for (int b = 0; b < L.n_box; ++b)
      tma_load_3d(sQ + (uint32_t)b * L.box_rows * kRowBytes, &map_q, &bars->tma_q, 0,
                  b * L.box_rows, bh);
    for (int b = 0; b < L.n_box; ++b) {
      const uint32_t off = (uint32_t)b * L.box_rows * kRowBytes;
      tma_load_3d(sK + off, &map_k, &bars->tma_kv, 0, b * L.box_rows, bh);
      tma_load_3d(sV + off, &map_v, &bars->tma_kv, 0, b * L.box_rows, bh);
    }
  }
  pdl_trigger();
  bool ok = fused_wait(&bars->tma_q, 0, abort, true);

  // ---- 1. the agents: given ones (bf16 [H][k][d] per batch set) or pooled
  // from the staged Q; thread per (agent row of the 128-row tile, 8-channel group)
  const __nv_bfloat16* ag_rows =
      agents ? agents + (long long)(bh / H) * ag_bstride + (long long)(bh % H) * k * d : nullptr;
  for (int it = threadIdx.x; it < kFusedMaxAgents * 8; it += kFusedThreads) {
    const int a = it >> 3, g = it & 7;
    if (ag_rows) {
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (a < k && g < groups)
        w = __ldg(reinterpret_cast<const uint4*>(ag_rows + (long long)a * d + g * 8));
      *reinterpret_cast<uint4*>(sA + a * kRowBytes + ((g ^ (a & 7)) << 4)) = w;
      continue;
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (ok && a < k && g < groups) {
      // adaptive bins [floor(i G / P), ceil((i + 1) G / P)) in 32-bit
      // arithmetic (grid sides <= 256 here)
      const int py = a / pool_w, px = a - py * pool_w;
      const int y0 = (py * grid_h) / pool_h, y1 = ((py + 1) * grid_h + pool_h - 1) / pool_h;
      const int x0 = (px * grid_w) / pool_w, x1 = ((px + 1) * grid_w + pool_w - 1) / pool_w;
      for (int y = y0; y < y1; ++y)
        for (int x = x0; x < x1; ++x) {
          const int r = y * grid_w + x;
          const uint4 w = *reinterpret_cast<const uint4*>(sQ + r * kRowBytes + ((g ^ (r & 7)) << 4));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] += bf16x2_lo(ws[i]);
            acc[2 * i + 1] += bf16x2_hi(ws[i]);
          }
        }
      const float inv = 1.f / (float)((y1 - y0) * (x1 - x0));
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= inv;
    }
    // rows >= k and channels >= d are zero: they pad the MMA's M and K
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(sA + a * kRowBytes + ((g ^ (a & 7)) << 4)) = o;
  }
  fence_proxy_async_smem();
  ok = fused_wait(&bars->tma_kv, 0, abort, ok);

  // ---- 2. S1 = A K^T (M = 128 agents, N = npad keys)
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(128, npad, 0, 0);
    for (int kk = 0; kk < d16; ++kk)
      mma_ss(tmem, sw128_desc(smem_u32(sA) + kk * 32, 16), sw128_desc(smem_u32(sK) + kk * 32, 16),
             idesc, kk > 0);
    mma_commit(&bars->mma);
  }
  ok = fused_wait(&bars->mma, 0, abort, ok);
  tc_fence_after();

  // slab of this warp: 16 TMEM lanes = rows, all columns
  const int quad = warp & 3;
  const int slab = quad * 32 + ((warp >> 2) & 1) * 16;
  const int j4 = lane & 3;
  const int r0 = slab + (lane >> 2), r1 = r0 + 8;
  const uint32_t lane_col = tmem + ((uint32_t)slab << 16);

  // ---- 3. softmax of the agent rows over the N keys; P1 over S1
  float l0 = 0.f, l1 = 0.f;
  {
    // slabs whose 16 rows are all padding agents (>= k) skip the work: their
    // U rows are never read
    const bool run = ok && slab < k;
    float t0 = -INFINITY, t1 = -INFINITY;
    if (run) {
      bc_slab_max(lane_col, N, npad, j4, t0, t1);
      t0 = row4_max(t0) * c;
      t1 = row4_max(t1) * c;
    }
    bc_slab_exp(lane_col, N, npad, j4, false, c, -t0, -t1, l0, l1, run, bars->chunk);
    l0 = row4_sum(l0);
    l1 = row4_sum(l1);
  }
  tc_fence_before();
  __syncthreads();

  // ---- 4. U = P1 V (M = 128 agents, N = dn, K = npad keys) into [128, 128 + dn)
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(128, dn, 0, 1);
    for (int kk = 0; kk < npad / 16; ++kk)   // keys [16 kk, 16 kk + 16)
      mma_ts(tmem + 128, tmem + bc_p_col(kk >> 2, false) + (kk & 3) * 8,
             sw128_desc(smem_u32(sV) + kk * 2048, (uint32_t)L.tensor_bytes), idesc, kk > 0);
    mma_commit(&bars->mma);
  }
  ok = fused_wait(&bars->mma, 1, abort, ok);
  tc_fence_after();

  // ---- 5. V_A = U / l1 -> bf16 rows of the MN-major operand (over K)
  {
    const float inv0 = r0 < k ? 1.f / l0 : 0.f, inv1 = r1 < k ? 1.f / l1 : 0.f;
    float u[32];                             // the 64 columns [128, 192): U and beyond
    if (ok && slab < k) {
      slab_ld64(lane_col + 128, u);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = 0.f;
    }
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {         // 8-column chunk
      const bool live = ch < groups;
      const uint32_t w0 = (live && r0 < k) ? pack_bf16x2(u[4 * ch] * inv0, u[4 * ch + 1] * inv0) : 0u;
      const uint32_t w1 =
          (live && r1 < k) ? pack_bf16x2(u[4 * ch + 2] * inv1, u[4 * ch + 3] * inv1) : 0u;
      *reinterpret_cast<uint32_t*>(sVA + r0 * kRowBytes + ((ch ^ (r0 & 7)) << 4) + j4 * 4) = w0;
      *reinterpret_cast<uint32_t*>(sVA + r1 * kRowBytes + ((ch ^ (r1 & 7)) << 4) + j4 * 4) = w1;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- 6. S2 = Q A^T per 128-query tile t into [128 t, 128 t + kpad)
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(128, kpad, 0, 0);
    for (int t = 0; t < n_qt; ++t)
      for (int kk = 0; kk < d16; ++kk)
        mma_ss(tmem + t * 128, sw128_desc(smem_u32(sQ) + t * kQTileBytes + kk * 32, 16),
               sw128_desc(smem_u32(sA) + kk * 32, 16), idesc, kk > 0);
    mma_commit(&bars->mma);
  }
  ok = fused_wait(&bars->mma, 0, abort, ok);
  tc_fence_after();

  float inv[2][2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    float m0 = 0.f, m1 = 0.f, s0 = 0.f, s1 = 0.f;
    if (t < n_qt) {
      // slabs whose rows are all past the slice's last query skip the work
      const bool run = ok && t * kQTile + slab < N;
      float a0 = -INFINITY, a1 = -INFINITY;
      if (run) {
        bc_slab_max(lane_col + t * 128, k, kpad, j4, a0, a1);
        m0 = row4_max(a0) * c;
        m1 = row4_max(a1) * c;
      }
      bc_slab_exp(lane_col + t * 128, k, kpad, j4, false, c, -m0, -m1, s0, s1, run, bars->chunk);
      s0 = row4_sum(s0);
      s1 = row4_sum(s1);
    }
    inv[t][0] = s0 > 0.f ? 1.f / s0 : 0.f;
    inv[t][1] = s1 > 0.f ? 1.f / s1 : 0.f;
  }
  tc_fence_before();
  __syncthreads();

  // ---- 7. O_t = P2_t V_A (M = 128 queries, N = dn, K = kpad agents) into
  // [128 t + 64, 128 t + 64 + dn)
  if (threadIdx.x == 0 && ok) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(128, dn, 0, 1);
    for (int t = 0; t < n_qt; ++t)
      for (int kk = 0; kk < kpad / 16; ++kk)
        mma_ts(tmem + t * 128 + 64, tmem + t * 128 + bc_p_col(kk >> 2, false) + (kk & 3) * 8,
               sw128_desc(smem_u32(sVA) + kk * 2048, kFusedMaxAgents * kRowBytes), idesc, kk > 0);
    mma_commit(&bars->mma);
  }
  ok = fused_wait(&bars->mma, 1, abort, ok);
  tc_fence_after();

  // epilogue: O / l2 -> bf16 -> swizzled staging tiles (over K and V) -> TMA
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (t >= n_qt) break;
    uint8_t* stage = sO + t * kQTileBytes;
    float o[32];                             // the 64 columns [128 t + 64, 128 t + 128): O_t
    if (ok && t * kQTile + slab < N) {
      slab_ld64(lane_col + t * 128 + 64, o);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0.f;
    }
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      if (ch < groups) {
        *reinterpret_cast<uint32_t*>(stage + r0 * kRowBytes + ((ch ^ (r0 & 7)) << 4) + j4 * 4) =
            pack_bf16x2(o[4 * ch] * inv[t][0], o[4 * ch + 1] * inv[t][0]);
        *reinterpret_cast<uint32_t*>(stage + r1 * kRowBytes + ((ch ^ (r1 & 7)) << 4) + j4 * 4) =
            pack_bf16x2(o[4 * ch + 2] * inv[t][1], o[4 * ch + 3] * inv[t][1]);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (ok && !*abort) {
      for (int t = 0; t < n_qt; ++t) tma_store_3d(&map_o, sO + t * kQTileBytes, 0, t * kQTile, bh);
      tma_store_commit();
    }
    tma_store_wait_read();                 // the staging may be released once read
    if (!ok) {
      // a wait gave up: let the staged copies and any MMA still running end
      // (bounded) before the CTA releases its TMEM and exits
      atomicOr(&g_watchdog, 1u);
      fused_drain_wait(&bars->tma_q, 0);
      fused_drain_wait(&bars->tma_kv, 0);
    }
    mma_commit(&bars->drain);
    fused_drain_wait(&bars->drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kFusedTmemCols);
  }
}

}  // namespace tc

// Host launch of the fused small-slice forward pass (no bias): pooled agents
// (agents = null) or given bf16 agents [H][n_agents][d] per batch set
// (ag_bstride elements between sets, 0 = shared over the batch).
inline cudaError_t tc_launch_fused_small(const void* q, const void* k, const void* v, void* out,
                                         int B, int H, int N, int d, int grid_h, int grid_w,
                                         int pool_h, int pool_w, int n_agents,
                                         const void* agents, long long ag_bstride, float c,
                                         cudaStream_t st) {
  using namespace tc;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL) return cudaErrorInvalidValue;
  const FusedLayout L = fused_layout(N);
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_3d(&mq, q, d, N, BH, L.box_rows) || !make_map_3d(&mk, k, d, N, BH, L.box_rows) ||
      !make_map_3d(&mv, v, d, N, BH, L.box_rows) || !make_map_3d(&mo, out, d, N, BH, kQTile))
    return cudaErrorInvalidValue;
  static std::atomic<int> flags[64];
  cudaError_t e = ensure_tc_smem(reinterpret_cast<const void*>(agent_fused_small_tc_kernel),
                                 (int)L.smem, flags);
  if (e != cudaSuccess) return e;
  return launch_kernel(agent_fused_small_tc_kernel, dim3((unsigned)BH), dim3(kFusedThreads),
                       L.smem, st, false, mq, mk, mv, mo, N, d, grid_h, grid_w, pool_h, pool_w,
                       n_agents, H, static_cast<const __nv_bfloat16*>(agents), ag_bstride, c);
}

}  // namespace aa
