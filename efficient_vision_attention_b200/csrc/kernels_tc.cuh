// Tensor-core kernels of the Agent Attention forward pass for bf16 inputs,
// head dim d <= 64, k <= 256 agents (sm_100a: tcgen05 MMA with TMEM
// accumulators, TMA tile loads/stores, mbarrier pipelines).
//
// Both stages are one "online-softmax attention" of a block of rows against a
// stream of columns, with the score tile and the output accumulator in TMEM:
//
//  agent_aggregate_tc  rows = agents (M = 128 per TMEM tile, 1 or 2 tiles),
//                      columns = keys streamed in tiles of 64 through an
//                      8-deep TMA ring of K and V tiles.  S = A K^T (SS MMA),
//                      online softmax in registers (one thread per agent row),
//                      P written back into TMEM as bf16 over S, U += P V (TS
//                      MMA, V as an MN-major operand) and l += P 1 (TS MMA
//                      against a tile of ones: the row sums come from the
//                      tensor core, summed from the same bf16 P).  Score tiles
//                      are double-buffered per softmax group, so the tensor
//                      core computes tile i+1 while the group works on tile i.
//                      A persistent grid cuts the key tiles of all slices into
//                      equal contiguous ranges (one range per CTA, one CTA per
//                      SM); each CTA writes one partial (U, running max,
//                      running sum) per slice it touches, merged afterwards by
//                      agent_merge_kernel.
//  agent_broadcast_tc  rows = queries streamed in tiles of 128 (TMA ring),
//                      columns = the k agents, resident in shared memory with
//                      V_A for the whole slice.  S = Q A^T, row softmax over k
//                      in registers, O = P V_A and l = P 1 on the tensor core,
//                      1/l applied in the epilogue, O staged in shared memory
//                      and written with TMA stores.
//
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and
// issues the MMAs (one thread), warps 2-5 and 6-9 are two softmax groups of
// 128 threads (thread = TMEM lane = row) working on alternating tiles (or, for
// k > 128 in the aggregation, on the two 128-agent halves).  Every wait is
// bounded; a wait that gives up makes its CTA skip the rest of its work and
// raises the device watchdog.
#pragma once

#include <atomic>

#include "common.cuh"
#include "tc_primitives.cuh"

namespace aa {

namespace tc {

constexpr int kThreads = 320;
constexpr int kRowBytes = 128;               // one swizzled 128-byte row per token (d <= 64 bf16)
constexpr int kKeyTile = 64;                 // keys per aggregation tile
constexpr int kQTile = 128;                  // queries per broadcast tile (MMA M)
constexpr int kKTileBytes = kKeyTile * kRowBytes;
constexpr int kQTileBytes = kQTile * kRowBytes;
constexpr int kAggStages = 8;
constexpr int kBcStages = 4;
constexpr int kMaxAgents = 256;
constexpr int kOnesBytes = 16 * kRowBytes;   // 16 rows of bf16 ones (row-sum operand)
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale only when the max grows by > 2^8

struct AggParams {
  int H, N, d, k;
  float c;                   // scale * log2(e)
  int tiles_per_slice;
  long long total_tiles;
  int ctas;
  int slots;                 // partial slots per slice
  float* part_u;             // [BH][slots][k][d]
  float* part_ml;            // [BH][slots][k][2]
};

struct BcParams {
  int H, N, d, k;
  float c;
  int tiles_per_slice;
  long long total_tiles;
  int ctas;
};

struct AggBars {
  uint64_t full[kAggStages], empty[kAggStages];
  uint64_t a_full, a_empty;
  uint64_t s_full[2][2], p_full[2][2], pv_done[2][2];   // [group][score buffer]
  uint64_t x_pub, x_done;    // group 1 -> group 0 hand-over per segment (k <= 128)
  uint32_t tmem_base;
  int abort;
  float m_x[128];
};

struct BcBars {
  uint64_t q_full[kBcStages], q_empty[kBcStages];
  uint64_t ag_full, ag_empty;
  uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ constexpr int round16(int x) { return (x + 15) & ~15; }

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Agent set coordinates (h, b) of slice bh for the 4-D agents tensor map.
__device__ __forceinline__ void agent_coords(long long bh, int H, int b_sets, int* h, int* b) {
  *h = (int)(bh % H);
  *b = b_sets > 1 ? (int)(bh / H) : 0;
}

// Fill the row-sum operand (16 rows x 128 bytes of bf16 1.0) and make it
// visible to the tensor core.
__device__ __forceinline__ void fill_ones(uint8_t* ones) {
  for (int i = threadIdx.x; i < kOnesBytes / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(ones)[i] = 0x3F803F80u;
  fence_proxy_async_smem();
}

// ============================================================== aggregation
constexpr size_t kAggSmemBytes = 1024 + (size_t)kMaxAgents * kRowBytes +
                                 2 * (size_t)kAggStages * kKTileBytes + kOnesBytes +
                                 sizeof(AggBars);

__global__ void __launch_bounds__(kThreads, 1)
    agent_aggregate_tc_kernel(const __grid_constant__ CUtensorMap map_k,
                              const __grid_constant__ CUtensorMap map_v,
                              const __grid_constant__ CUtensorMap map_a, int a_sets,
                              AggParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sK = sA + kMaxAgents * kRowBytes;
  uint8_t* sV = sK + kAggStages * kKTileBytes;
  uint8_t* sOnes = sV + kAggStages * kKTileBytes;
  AggBars* bars = reinterpret_cast<AggBars*>(sOnes + kOnesBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long cta = blockIdx.x;
  const long long t_begin = (cta * p.total_tiles) / p.ctas;
  const long long t_end = ((cta + 1) * p.total_tiles) / p.ctas;
  const int tps = p.tiles_per_slice;
  const bool two = p.k > 128;                 // two 128-row agent tiles
  const int d16 = (p.d + 15) >> 4;            // K steps of S = A K^T
  const int dn = d16 * 16;                    // N of U += P V; l sits in column dn

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAggStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->a_full, 1);
    mbar_init(&bars->a_empty, 1);
    for (int g = 0; g < 2; ++g)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&bars->s_full[g][b], 1);
        mbar_init(&bars->p_full[g][b], 128);
        mbar_init(&bars->pv_done[g][b], 1);
      }
    mbar_init(&bars->x_pub, 128);
    mbar_init(&bars->x_done, 128);
    bars->abort = 0;
    mbar_fence_init();
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_a);
  }
  fill_ones(sOnes);
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // TMEM columns: score buffer b of group g at g*128 + b*64 (P over its first
  // 32 columns), U of group g at 256 + g*128 (dn columns), l at 256 + g*128 + dn.

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      long long it = 0;
      int seg = 0;
      const uint32_t a_bytes = (two ? 256 : 128) * kRowBytes;
      for (long long t = t_begin; t < t_end; ++seg) {
        const long long bh = t / tps;
        const long long seg_end = min(t_end, (bh + 1) * tps);
        if (seg > 0 && !mbar_wait(&bars->a_empty, (seg - 1) & 1, abort)) break;
        int h, b;
        agent_coords(bh, p.H, a_sets, &h, &b);
        mbar_expect_tx(&bars->a_full, a_bytes);
        tma_load_4d(sA, &map_a, &bars->a_full, 0, 0, h, b);
        bool ok = true;
        for (; t < seg_end; ++t, ++it) {
          const int s = (int)(it % kAggStages);
          if (it >= kAggStages &&
              !mbar_wait(&bars->empty[s], (uint32_t)((it / kAggStages) - 1) & 1, abort)) {
            ok = false;
            break;
          }
          const int key0 = (int)(t - bh * tps) * kKeyTile;
          mbar_expect_tx(&bars->full[s], 2 * kKTileBytes);
          tma_load_3d(sK + s * kKTileBytes, &map_k, &bars->full[s], 0, key0, (int)bh);
          tma_load_3d(sV + s * kKTileBytes, &map_v, &bars->full[s], 0, key0, (int)bh);
        }
        if (!ok) break;
      }
      // On abort, wait (bounded) for the loads already issued before leaving.
      if (*abort) {
        for (long long j = (it > kAggStages ? it - kAggStages : 0); j < it; ++j) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars->full[j % kAggStages], (uint32_t)(j / kAggStages) & 1) &&
                 globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t idesc_s = idesc_bf16(128, kKeyTile, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, dn, 0, 1);
      const uint32_t idesc_l = idesc_bf16(128, 16, 0, 1);
      const uint32_t sA_addr = smem_u32(sA), sK_addr = smem_u32(sK), sV_addr = smem_u32(sV);
      const uint64_t ones_desc = sw128_desc(smem_u32(sOnes), 8192);
      long long it0 = 0;
      int seg = 0;
      int cnt_s[2] = {0, 0}, cnt_p[2] = {0, 0};
      bool ok = true;
      for (long long t = t_begin; t < t_end && ok; ++seg) {
        const long long bh = t / tps;
        const long long seg_end = min(t_end, (bh + 1) * tps);
        const int n = (int)(seg_end - t);
        if (!mbar_wait(&bars->a_full, seg & 1, abort)) break;
        tc_fence_after();
        bool first[2] = {true, true};
        auto issue_s = [&](int i) -> bool {
          const long long itg = it0 + i;
          const int s = (int)(itg % kAggStages);
          if (!mbar_wait(&bars->full[s], (uint32_t)(itg / kAggStages) & 1, abort)) return false;
          tc_fence_after();
          for (int g = 0; g < 2; ++g) {
            if (!two && (i & 1) != g) continue;
            const int J = cnt_s[g], b = J & 1;
            if (J >= 2) {   // the buffer's previous P has been consumed
              if (!mbar_wait(&bars->pv_done[g][b], (uint32_t)((J >> 1) - 1) & 1, abort))
                return false;
              tc_fence_after();
            }
            const int mt = two ? g : 0;
            const uint32_t d_tm = tmem + g * 128 + b * 64;
            for (int kk = 0; kk < d16; ++kk) {
              const uint64_t da = sw128_desc(sA_addr + mt * 128 * kRowBytes + kk * 32, 16);
              const uint64_t db = sw128_desc(sK_addr + s * kKTileBytes + kk * 32, 16);
              mma_ss(d_tm, da, db, idesc_s, kk > 0);
            }
            mma_commit(&bars->s_full[g][b]);
            ++cnt_s[g];
          }
          return true;
        };
        auto issue_pv = [&](int i) -> bool {
          const long long itg = it0 + i;
          const int s = (int)(itg % kAggStages);
          for (int g = 0; g < 2; ++g) {
            if (!two && (i & 1) != g) continue;
            const int J = cnt_p[g], b = J & 1;
            if (!mbar_wait(&bars->p_full[g][b], (uint32_t)(J >> 1) & 1, abort)) return false;
            tc_fence_after();
            const uint32_t p_tm = tmem + g * 128 + b * 64;
            const uint32_t u_tm = tmem + 256 + g * 128;
            for (int kk = 0; kk < kKeyTile / 16; ++kk) {
              const uint32_t acc = (!first[g] || kk > 0) ? 1u : 0u;
              const uint64_t dv = sw128_desc(sV_addr + s * kKTileBytes + kk * 2048, 8192);
              mma_ts(u_tm, p_tm + kk * 8, dv, idesc_pv, acc);
              mma_ts(u_tm + dn, p_tm + kk * 8, ones_desc, idesc_l, acc);
            }
            first[g] = false;
            mma_commit(&bars->pv_done[g][b]);
            ++cnt_p[g];
          }
          mma_commit(&bars->empty[s]);
          return true;
        };
        // one tile of look-ahead: S of tile i is issued before P V of tile i-1
        for (int i = 0; i < n && ok; ++i) {
          ok = issue_s(i);
          if (ok && i > 0) ok = issue_pv(i - 1);
        }
        if (ok) ok = issue_pv(n - 1);
        mma_commit(&bars->a_empty);
        it0 += n;
        t = seg_end;
      }
      // Let every MMA issued so far finish before TMEM is released.
      mma_commit(&bars->a_full);   // a_full is no longer waited on: use it as a drain marker
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&bars->a_full, (uint32_t)seg & 1) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // ---------------------------------------------------- softmax groups
    // Every thread walks the same segments and tiles whatever happens; after a
    // failed (timed-out) wait it only skips work, so no barrier is left short.
    const int g = (warp - 2) >> 2;            // group 0: warps 2-5, group 1: warps 6-9
    const int quad = warp & 3;                // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;         // TMEM lane = row of the 128-row tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t u_col = tmem + lane_off + 256 + g * 128;
    const int agent = (two ? g * 128 : 0) + row;
    const bool warp_active = (two ? g * 128 : 0) + quad * 32 < p.k;
    int J = 0, seg = 0;
    bool ok = true;
    for (long long t = t_begin; t < t_end; ++seg) {
      const long long bh = t / tps;
      const long long seg_end = min(t_end, (bh + 1) * tps);
      const int n = (int)(seg_end - t);
      const int n_mine = two ? n : (g == 0 ? (n + 1) / 2 : n / 2);
      float m = -INFINITY;
      bool first = true;
      for (int i = 0; i < n; ++i) {
        if (!two && (i & 1) != g) continue;
        const int b = J & 1;
        const uint32_t s_col = tmem + lane_off + g * 128 + b * 64;
        const int valid = min(kKeyTile, p.N - (int)(t + i - bh * tps) * kKeyTile);
        if (ok) ok = warp_wait(&bars->s_full[g][b], (uint32_t)(J >> 1) & 1, abort);
        tc_fence_after();
        if (ok && warp_active) {
          float v[64];
          tmem_ld64(s_col, v);
          if (valid < kKeyTile) {               // ragged last tile: mask the missing keys
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (e >= valid) v[e] = -INFINITY;
          }
          float (&v0)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
          float (&v1)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
          const float mt = max32(v1, max32(v0, -INFINITY)) * p.c;
          if (first) {
            m = mt;
            first = false;
          } else if (__any_sync(0xffffffffu, mt > m + kRescaleThreshold)) {
            // the running max grew a lot: once the previous P V has landed,
            // rescale U and l by 2^(m_old - m_new)
            ok = warp_wait(&bars->pv_done[g][(J - 1) & 1], (uint32_t)((J - 1) >> 1) & 1, abort);
            tc_fence_after();
            if (ok) {
              const float m_new = fmaxf(m, mt);
              const float alpha = ex2(m - m_new);
              m = m_new;
#pragma unroll 1
              for (int c = 0; c < dn / 16 + 1; ++c) {
                float u[16];
                tmem_ld16(u_col + c * 16, u);
#pragma unroll
                for (int e = 0; e < 16; ++e) u[e] *= alpha;
                tmem_st16(u_col + c * 16, u);
              }
            }
          }
          if (ok) {
            uint32_t pk[16];
            exp_pack32(v0, p.c, -m, pk);
            tmem_st16u(s_col, pk);
            exp_pack32(v1, p.c, -m, pk);
            tmem_st16u(s_col + 16, pk);
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->p_full[g][b]);
        ++J;
      }
      // ---- segment epilogue: write this CTA's partial for slice bh
      const int slot = (int)(cta - ((bh * tps + 1) * p.ctas - 1) / p.total_tiles);
      const long long slot_row = (bh * p.slots + slot) * (long long)p.k;
      if (n_mine > 0 && ok)
        ok = warp_wait(&bars->pv_done[g][(J - 1) & 1], (uint32_t)((J - 1) >> 1) & 1, abort);
      tc_fence_after();
      if (two) {
        if (ok && warp_active) {            // warp-uniform: the TMEM loads are warp-collective
          const bool mine = agent < p.k;
          const float l = tmem_ld1(u_col + dn);
          float* dst = p.part_u + (slot_row + agent) * p.d;
#pragma unroll 1
          for (int c = 0; c < dn / 16; ++c) {
            float u[16];
            tmem_ld16(u_col + c * 16, u);
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              if (mine && c * 16 + e < p.d)
                *reinterpret_cast<float4*>(dst + c * 16 + e) =
                    make_float4(u[e], u[e + 1], u[e + 2], u[e + 3]);
          }
          if (mine) {
            p.part_ml[(slot_row + agent) * 2] = m;
            p.part_ml[(slot_row + agent) * 2 + 1] = l;
          }
        }
      } else if (g == 1) {
        // both groups hold the same agent rows over different key tiles:
        // group 1 publishes its running max and waits until group 0 has read
        // its accumulators
        if (n_mine > 0 && ok && warp_active && row < p.k) bars->m_x[row] = m;
        tc_fence_before();
        mbar_arrive(&bars->x_pub);
        if (ok) ok = warp_wait(&bars->x_done, (uint32_t)seg & 1, abort);
        tc_fence_after();
      } else {
        if (ok) ok = warp_wait(&bars->x_pub, (uint32_t)seg & 1, abort);
        tc_fence_after();
        if (ok && warp_active) {            // warp-uniform: the TMEM loads are warp-collective
          const bool mine = row < p.k;
          const bool has1 = (n / 2) > 0;
          const uint32_t u1_col = tmem + lane_off + 256 + 128;
          float mm = m, a0 = 1.f, a1 = 0.f;
          if (has1 && mine) {
            const float m1 = bars->m_x[row];
            mm = fmaxf(m, m1);
            a0 = ex2(m - mm);
            a1 = ex2(m1 - mm);
          }
          float l = a0 * tmem_ld1(u_col + dn);
          if (has1) l += a1 * tmem_ld1(u1_col + dn);
          float* dst = p.part_u + (slot_row + row) * p.d;
#pragma unroll 1
          for (int c = 0; c < dn / 16; ++c) {
            float u[16];
            tmem_ld16(u_col + c * 16, u);
            if (has1) {
              float w[16];
              tmem_ld16(u1_col + c * 16, w);
#pragma unroll
              for (int e = 0; e < 16; ++e) u[e] = a0 * u[e] + a1 * w[e];
            }
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              if (mine && c * 16 + e < p.d)
                *reinterpret_cast<float4*>(dst + c * 16 + e) =
                    make_float4(u[e], u[e + 1], u[e + 2], u[e + 3]);
          }
          if (mine) {
            p.part_ml[(slot_row + row) * 2] = mm;
            p.part_ml[(slot_row + row) * 2 + 1] = l;
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->x_done);
      }
      t = seg_end;
    }
    if (!ok) *abort = 1;
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================ broadcast
constexpr size_t kBcSmemBytes = 1024 + 2 * (size_t)kMaxAgents * kRowBytes +
                                (size_t)kBcStages * kQTileBytes + 2 * (size_t)kQTileBytes +
                                kOnesBytes + sizeof(BcBars);

// Row max over the first kpad columns of a score row (columns >= k masked).
// 64 columns per TMEM load; kpad (a multiple of 16) may end in a 32- or
// 16-column remainder.
__device__ __forceinline__ float bc_row_max(uint32_t s_col, int k, int kpad) {
  float mx = -INFINITY;
  int c = 0;
#pragma unroll 1
  for (; c + 64 <= kpad; c += 64) {
    float v[64];
    tmem_ld64(s_col + c, v);
    if (c + 64 > k) {
#pragma unroll
      for (int e = 0; e < 64; ++e)
        if (c + e >= k) v[e] = -INFINITY;
    }
    mx = max32(*reinterpret_cast<float(*)[32]>(&v[0]),
               max32(*reinterpret_cast<float(*)[32]>(&v[32]), mx));
  }
#pragma unroll 1
  for (; c < kpad; c += 32) {
    float v[32];
    if (c + 32 <= kpad) {
      tmem_ld32(s_col + c, v);
    } else {                      // a 16-column remainder
      float h[16];
      tmem_ld16(s_col + c, h);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        v[e] = h[e];
        v[16 + e] = -INFINITY;
      }
    }
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (c + e >= k) v[e] = -INFINITY;
    mx = max32(v, mx);
  }
  return mx;
}

// P = 2^(S*c - m) as bf16 over the first kpad/2 columns (columns >= k give 0).
__device__ __forceinline__ void bc_row_exp(uint32_t s_col, int k, int kpad, float c_scale,
                                           float m) {
  int c = 0;
#pragma unroll 1
  for (; c + 64 <= kpad; c += 64) {
    float v[64];
    tmem_ld64(s_col + c, v);
    if (c + 64 > k) {
#pragma unroll
      for (int e = 0; e < 64; ++e)
        if (c + e >= k) v[e] = -INFINITY;
    }
    uint32_t pk[16];
    exp_pack32(*reinterpret_cast<float(*)[32]>(&v[0]), c_scale, -m, pk);
    tmem_st16u(s_col + c / 2, pk);
    exp_pack32(*reinterpret_cast<float(*)[32]>(&v[32]), c_scale, -m, pk);
    tmem_st16u(s_col + c / 2 + 16, pk);
  }
#pragma unroll 1
  for (; c < kpad; c += 32) {
    float v[32];
    uint32_t pk[16];
    if (c + 32 <= kpad) {
      tmem_ld32(s_col + c, v);
    } else {
      float h[16];
      tmem_ld16(s_col + c, h);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        v[e] = h[e];
        v[16 + e] = -INFINITY;
      }
    }
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (c + e >= k) v[e] = -INFINITY;
    exp_pack32(v, c_scale, -m, pk);
    if (c + 32 <= kpad) {
      tmem_st16u(s_col + c / 2, pk);
    } else {
      uint32_t lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = pk[e];
      tmem_st8(s_col + c / 2, lo);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    agent_broadcast_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                              const __grid_constant__ CUtensorMap map_a,
                              const __grid_constant__ CUtensorMap map_va,
                              const __grid_constant__ CUtensorMap map_o, int a_sets,
                              BcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sVA = sA + kMaxAgents * kRowBytes;
  uint8_t* sQ = sVA + kMaxAgents * kRowBytes;
  uint8_t* sO = sQ + kBcStages * kQTileBytes;
  uint8_t* sOnes = sO + 2 * kQTileBytes;
  BcBars* bars = reinterpret_cast<BcBars*>(sOnes + kOnesBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long cta = blockIdx.x;
  const long long t_begin = (cta * p.total_tiles) / p.ctas;
  const long long t_end = ((cta + 1) * p.total_tiles) / p.ctas;
  const int tps = p.tiles_per_slice;
  const int n_tiles = (int)(t_end - t_begin);
  const int kpad = round16(p.k);
  const int d16 = (p.d + 15) >> 4;
  const int dn = d16 * 16;
  const int o_col = ((kpad / 2) + 31) & ~31;   // O accumulator column inside a 256-column buffer

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBcStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    mbar_init(&bars->ag_full, 1);
    mbar_init(&bars->ag_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_free[i], 128);
    }
    bars->abort = 0;
    mbar_fence_init();
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_va);
    prefetch_tensormap(&map_o);
  }
  fill_ones(sOnes);
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // TMEM: buffer b at column b*256: S over [0, kpad), P (bf16) over [0, kpad/2),
  // O over [o_col, o_col + dn), l at o_col + dn.

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      long long cur = -1;
      int n_slices = 0;
      const uint32_t ag_bytes = 2u * kpad * kRowBytes;
      int j = 0;
      for (; j < n_tiles; ++j) {
        const long long t = t_begin + j;
        const long long bh = t / tps;
        if (bh != cur) {
          if (n_slices > 0 && !mbar_wait(&bars->ag_empty, (n_slices - 1) & 1, abort)) break;
          int h, b;
          agent_coords(bh, p.H, a_sets, &h, &b);
          mbar_expect_tx(&bars->ag_full, ag_bytes);
          tma_load_4d(sA, &map_a, &bars->ag_full, 0, 0, h, b);
          tma_load_3d(sVA, &map_va, &bars->ag_full, 0, 0, (int)bh);
          cur = bh;
          ++n_slices;
        }
        const int s = j % kBcStages;
        if (j >= kBcStages && !mbar_wait(&bars->q_empty[s], ((j / kBcStages) - 1) & 1, abort))
          break;
        mbar_expect_tx(&bars->q_full[s], kQTileBytes);
        tma_load_3d(sQ + s * kQTileBytes, &map_q, &bars->q_full[s], 0,
                    (int)(t - bh * tps) * kQTile, (int)bh);
      }
      if (*abort) {
        for (int i = (j > kBcStages ? j - kBcStages : 0); i < j; ++i) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars->q_full[i % kBcStages], (uint32_t)(i / kBcStages) & 1) &&
                 globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t idesc_s = idesc_bf16(128, kpad, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, dn, 0, 1);
      const uint32_t idesc_l = idesc_bf16(128, 16, 0, 1);
      const uint32_t sA_addr = smem_u32(sA), sVA_addr = smem_u32(sVA), sQ_addr = smem_u32(sQ);
      const uint64_t ones_desc = sw128_desc(smem_u32(sOnes), 8192);
      int n_slices = 0;
      long long cur = -1;
      auto slice_of = [&](int j) { return (t_begin + j) / tps; };
      auto issue_s = [&](int j) -> bool {
        const int b = j & 1;
        if (slice_of(j) != cur) {
          if (!mbar_wait(&bars->ag_full, n_slices & 1, abort)) return false;
          cur = slice_of(j);
          ++n_slices;
        }
        if (j >= 2 && !mbar_wait(&bars->o_free[b], ((j >> 1) - 1) & 1, abort)) return false;
        const int s = j % kBcStages;
        if (!mbar_wait(&bars->q_full[s], (j / kBcStages) & 1, abort)) return false;
        tc_fence_after();
        for (int kk = 0; kk < d16; ++kk) {
          const uint64_t da = sw128_desc(sQ_addr + s * kQTileBytes + kk * 32, 16);
          const uint64_t db = sw128_desc(sA_addr + kk * 32, 16);
          mma_ss(tmem + b * 256, da, db, idesc_s, kk > 0);
        }
        mma_commit(&bars->s_full[b]);
        mma_commit(&bars->q_empty[s]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int b = j & 1;
        if (!mbar_wait(&bars->p_full[b], (j >> 1) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t o_tm = tmem + b * 256 + o_col;
        for (int kk = 0; kk < kpad / 16; ++kk) {
          const uint32_t p_tm = tmem + b * 256 + kk * 8;
          mma_ts(o_tm, p_tm, sw128_desc(sVA_addr + kk * 2048, 8192), idesc_pv, kk > 0);
          mma_ts(o_tm + dn, p_tm, ones_desc, idesc_l, kk > 0);
        }
        mma_commit(&bars->o_full[b]);
        if (j + 1 == n_tiles || slice_of(j + 1) != slice_of(j)) mma_commit(&bars->ag_empty);
        return true;
      };
      bool ok = n_tiles > 0 ? issue_s(0) : true;
      for (int j = 0; j < n_tiles && ok; ++j) {
        const bool next_same = j + 1 < n_tiles && slice_of(j + 1) == slice_of(j);
        if (next_same) {
          ok = issue_s(j + 1);
          if (ok) ok = issue_pv(j);
        } else {
          ok = issue_pv(j);
          if (ok && j + 1 < n_tiles) ok = issue_s(j + 1);
        }
      }
      // drain: all MMAs complete before TMEM is released
      mma_commit(&bars->ag_full);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&bars->ag_full, (uint32_t)n_slices & 1) &&
             globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // ------------------------------------------- softmax + epilogue groups
    const int g = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t s_col = tmem + lane_off + g * 256;
    const uint32_t o_tm = s_col + o_col;
    uint8_t* stage = sO + g * kQTileBytes;
    const bool leader = (warp == 2 + 4 * g) && lane == 0;
    bool ok = true;
    for (int j = g; j < n_tiles; j += 2) {
      const int u = j >> 1;
      const long long t = t_begin + j;
      const long long bh = t / tps;
      const int q0 = (int)(t - bh * tps) * kQTile;
      if (ok) ok = warp_wait(&bars->s_full[g], u & 1, abort);
      tc_fence_after();
      if (ok) {
        const float m = bc_row_max(s_col, p.k, kpad) * p.c;
        bc_row_exp(s_col, p.k, kpad, p.c, m);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bars->p_full[g]);
      // epilogue: O = (P V_A) / (P 1) -> bf16 -> swizzled staging tile -> TMA store
      if (ok) ok = warp_wait(&bars->o_full[g], u & 1, abort);
      tc_fence_after();
      float o[64];
      float l = 1.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (ok && c * 32 < dn) {
          float v[32];
          if (c * 32 + 32 <= dn) {
            tmem_ld32(o_tm + c * 32, v);
          } else {
            float h[16];
            tmem_ld16(o_tm + c * 32, h);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              v[e] = h[e];
              v[16 + e] = 0.f;
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) o[c * 32 + e] = v[e];
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[c * 32 + e] = 0.f;
        }
      }
      if (ok) l = tmem_ld1(o_tm + dn);
      tc_fence_before();
      mbar_arrive(&bars->o_free[g]);
      const float inv = 1.f / l;
      if (leader) tma_store_wait_read();
      named_barrier(3 + g, 128);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        if (ch * 8 < p.d) {
          uint4 w;
          w.x = pack_bf16x2(o[ch * 8 + 0] * inv, o[ch * 8 + 1] * inv);
          w.y = pack_bf16x2(o[ch * 8 + 2] * inv, o[ch * 8 + 3] * inv);
          w.z = pack_bf16x2(o[ch * 8 + 4] * inv, o[ch * 8 + 5] * inv);
          w.w = pack_bf16x2(o[ch * 8 + 6] * inv, o[ch * 8 + 7] * inv);
          *reinterpret_cast<uint4*>(stage + row * kRowBytes + ((ch ^ (row & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      named_barrier(3 + g, 128);
      if (leader && !*abort) {
        tma_store_3d(&map_o, stage, 0, q0, (int)bh);
        tma_store_commit();
      }
    }
    if (leader) tma_store_wait_all();
    if (!ok) *abort = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc

// ================================================================ host side
inline bool tc_supported(int d, int k) { return d >= 8 && d <= 64 && k >= 1 && k <= 256; }

inline void tc_plan_aggregate(long long BH, int N, int k, int sm_count, SplitPlan* plan) {
  (void)k;
  const int tps = (N + tc::kKeyTile - 1) / tc::kKeyTile;
  const long long total = BH * tps;
  const int ctas = (int)(total < sm_count ? total : sm_count);
  const long long min_per_cta = total / ctas;
  plan->fixed = 0;
  plan->ctas = ctas;
  plan->total_tiles = total;
  plan->tiles_per_slice = tps;
  plan->slots = (int)((tps + min_per_cta - 1) / min_per_cta + 1);
}

namespace tc {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> cached{nullptr};
  EncodeTiledFn fn = cached.load(std::memory_order_acquire);
  if (fn) return fn;
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  fn = reinterpret_cast<EncodeTiledFn>(ptr);
  cached.store(fn, std::memory_order_release);
  return fn;
}

// bf16 tensor [sets][rows][d] (row-major), box = 64 columns x box_rows rows,
// 128-byte swizzle, zero fill outside the tensor.
inline bool make_map_3d(CUtensorMap* map, const void* base, int d, long long rows, long long sets,
                        int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)sets};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Agents: slice (b, h) at base + b*batch_stride + h*k*d elements; 4-D map
// (d, k, H, B) with the batch dimension collapsed to 1 when it is shared.
inline bool make_map_agents(CUtensorMap* map, const void* base, int d, int k, int H, int B,
                            long long batch_stride, int box_rows, int* sets_out) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int sets = batch_stride > 0 ? B : 1;
  const long long bstride = batch_stride > 0 ? batch_stride : (long long)H * k * d;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)k, (cuuint64_t)H, (cuuint64_t)sets};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)k * d * 2, (cuuint64_t)bstride * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  *sets_out = sets;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline std::atomic<int>* smem_flags_agg() {
  static std::atomic<int> f[64];
  return f;
}
inline std::atomic<int>* smem_flags_bc() {
  static std::atomic<int> f[64];
  return f;
}

inline cudaError_t ensure_tc_smem(const void* kernel, int bytes, std::atomic<int>* flags) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && flags[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev < 64) flags[dev].store(bytes, std::memory_order_relaxed);
  return e;
}

}  // namespace tc

// Returns 0 on success, AA_ERR_CUDA-style codes through the callers.
inline cudaError_t tc_launch_aggregate(const void* agents, long long a_bstride, long long a_hstride,
                                       const void* k, const void* v, int B, int H, int N, int d,
                                       int n_agents, float c, const SplitPlan& plan,
                                       float* part_u, float* part_ml, cudaStream_t st) {
  (void)a_hstride;
  using namespace tc;
  CUtensorMap mk, mv, ma;
  int a_sets = 1;
  const long long BH = (long long)B * H;
  const int box_a = n_agents > 128 ? 256 : 128;
  if (!make_map_3d(&mk, k, d, N, BH, kKeyTile) || !make_map_3d(&mv, v, d, N, BH, kKeyTile) ||
      !make_map_agents(&ma, agents, d, n_agents, H, B, a_bstride, box_a, &a_sets))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_tc_smem(reinterpret_cast<const void*>(agent_aggregate_tc_kernel),
                                 (int)kAggSmemBytes, smem_flags_agg());
  if (e != cudaSuccess) return e;
  AggParams p;
  p.H = H;
  p.N = N;
  p.d = d;
  p.k = n_agents;
  p.c = c;
  p.tiles_per_slice = plan.tiles_per_slice;
  p.total_tiles = plan.total_tiles;
  p.ctas = plan.ctas;
  p.slots = plan.slots;
  p.part_u = part_u;
  p.part_ml = part_ml;
  agent_aggregate_tc_kernel<<<plan.ctas, kThreads, kAggSmemBytes, st>>>(mk, mv, ma, a_sets, p);
  return cudaGetLastError();
}

inline cudaError_t tc_launch_broadcast(const void* q, const void* agents, long long a_bstride,
                                       const void* va, void* out, int B, int H, int N, int d,
                                       int n_agents, float c, int sm_count, cudaStream_t st) {
  using namespace tc;
  CUtensorMap mq, ma, mva, mo;
  int a_sets = 1;
  const long long BH = (long long)B * H;
  const int kpad = round16(n_agents);
  if (!make_map_3d(&mq, q, d, N, BH, kQTile) || !make_map_3d(&mo, out, d, N, BH, kQTile) ||
      !make_map_3d(&mva, va, d, n_agents, BH, kpad) ||
      !make_map_agents(&ma, agents, d, n_agents, H, B, a_bstride, kpad, &a_sets))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_tc_smem(reinterpret_cast<const void*>(agent_broadcast_tc_kernel),
                                 (int)kBcSmemBytes, smem_flags_bc());
  if (e != cudaSuccess) return e;
  BcParams p;
  p.H = H;
  p.N = N;
  p.d = d;
  p.k = n_agents;
  p.c = c;
  p.tiles_per_slice = (N + kQTile - 1) / kQTile;
  p.total_tiles = BH * p.tiles_per_slice;
  p.ctas = (int)(p.total_tiles < sm_count ? p.total_tiles : sm_count);
  agent_broadcast_tc_kernel<<<p.ctas, kThreads, kBcSmemBytes, st>>>(mq, ma, mva, mo, a_sets, p);
  return cudaGetLastError();
}

}  // namespace aa
