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
//                      online softmax in registers, P written back into TMEM
//                      as bf16 over S, U += P V (TS MMA, V as an MN-major
//                      operand); the row sums are accumulated in registers.
//                      Score tiles are double-buffered per softmax group, so
//                      the tensor core computes tile i+1 while the group works
//                      on tile i.  A persistent grid cuts the key tiles of all
//                      slices into equal contiguous ranges (one range per CTA,
//                      one CTA per SM); each CTA writes one partial (U,
//                      running max, running sum) per slice it touches, merged
//                      afterwards by agent_merge_kernel.
//  agent_broadcast_tc  rows = queries streamed in tiles of 128 (TMA ring),
//                      columns = the k agents, resident in shared memory with
//                      V_A for the whole slice.  S = Q A^T, row softmax over k
//                      in registers, O = P V_A on the tensor core, 1/l applied
//                      in the epilogue, O staged in shared memory and written
//                      with TMA stores.
//
// Warp roles (608 threads): warp 0 issues TMA loads; warps 1 and 2 each issue
// the MMAs of one softmax group (one thread each: a single issuing thread
// spends about 57 cycles per tcgen05.mma, so two issuers double the MMA rate
// and keep the groups independent); warps 3-10 and 11-18 are the two softmax
// groups, working on alternating tiles (or, for k > 128 in the aggregation,
// on the two 128-agent halves).  In a group, TMEM lane = row, and each warp
// owns a 16-row slab of the 128 rows with all the columns of the tile (the
// 16x256b TMEM access shape spreads a row over 4 threads, which combine row
// maxima and sums with shuffles), so no warp waits for another inside the
// softmax of a tile.  Every wait
// is bounded; a wait that gives up makes its CTA skip the rest of its work
// and raises the device watchdog.
#pragma once

#include <atomic>

#include "common.cuh"
#include "tc_primitives.cuh"

namespace aa {

namespace tc {

constexpr int kSoftmaxThreads = 256;           // per softmax group: 8 warps, two per lane quadrant
constexpr int kFirstSoftmaxWarp = 3;
constexpr int kThreads = kFirstSoftmaxWarp * 32 + 2 * kSoftmaxThreads;
constexpr int kSoftmaxWarps = kSoftmaxThreads / 32;  // arrivals per group on its barriers
constexpr int kRowBytes = 128;               // one swizzled 128-byte row per token (d <= 64 bf16)
constexpr int kKeyTile = 64;                 // keys per aggregation tile
constexpr int kQTile = 128;                  // queries per broadcast tile (MMA M)
constexpr int kKTileBytes = kKeyTile * kRowBytes;
constexpr int kQTileBytes = kQTile * kRowBytes;
constexpr int kAggStages = 8;
constexpr int kSBuf = 3;                     // score buffers per aggregation group
constexpr int kBcStages = 4;
constexpr int kMaxAgents = 256;
constexpr int kAgentBufBytes = kMaxAgents * kRowBytes;   // one agent tile (all agents of a slice)
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale only when the max grows by > 2^8

// Agent bias in the score tiles: a dense fp16 copy of B * log2(e) (logits in
// log2 units), made per call from the row, column and block components.  B1
// (aggregation): [H][k][ld] with the tokens contiguous (ld >= N, even, zero
// past N); B2 (broadcast): [H][N][ld] with the agents contiguous (ld = k
// rounded up to 16, zero past k).  A thread's score column pair reads its two
// logits as one 32-bit word.
struct BiasParams {
  const __half* dense;       // null: no bias
  int ld;                    // row length of the dense copy, in elements
  __host__ __device__ bool any() const { return dense != nullptr; }
};

struct AggParams {
  int H, N, d, k;
  float c;                   // scale * log2(e)
  int tiles_per_slice;
  long long total_tiles;
  int ctas;
  int slots;                 // partial slots per slice
  float* part_u;             // [BH][slots][k][d]
  float* part_ml;            // [BH][slots][k][2]
  BiasParams bias;           // B1 (agents x keys), all null when absent
};

// Per-query statistics of the broadcast for the backward pass (the stats
// instantiation writes these instead of O): the row max of the scores in log2
// units (m), the row sum of 2^(s - m) (l), D = dO . O with O the normalised
// output row, and the row's 2^(s - m) themselves as bf16 (p).  dout
// [BH][N][d] bf16; m, l, D [BH][N] fp32; p [BH][N][kpad] bf16.
struct BcStats {
  const __nv_bfloat16* dout;
  float* m;
  float* l;
  float* D;
  __nv_bfloat16* p;          // [BH][N][kpad]: 2^(s - m) as bf16 (not normalised)
  // Column mode (the key side: the broadcast run over K): non-null col_ml
  // [BH][k][2] holds each agent's aggregation max (log2 units) and sum; the
  // pass then stores 2^(s - m_agent) for every (key, agent) into p and
  // nothing else (dout, m, l, D unused).
  const float* col_ml;
};

struct BcParams {
  int H, N, d, k;
  float c;
  int tiles_per_slice;
  long long total_tiles;
  int ctas;
  BiasParams bias;           // B2 (queries x agents), all null when absent
  BcStats stats;             // read only by the stats instantiation
};

struct AggBars {
  uint64_t full[kAggStages], empty[kAggStages];
  uint64_t a_full[2], a_empty[2];   // agent tile buffers, alternating per segment
  uint64_t s_full[2][kSBuf], p_full[2][kSBuf], pv_done[2][kSBuf];   // [group][score buffer]
  uint64_t x_pub, x_done;    // group 1 -> group 0 hand-over per segment (k <= 128)
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
  float m_x[128];            // group 1's row maxima and sums at a segment end (k <= 128)
  float l_x[128];
};

struct BcBars {
  uint64_t q_full[kBcStages], q_empty[kBcStages];
  uint64_t ag_full, ag_empty;
  uint64_t s_full[2], o_full[2], o_free[2];
  uint64_t p_chunk[2][4];    // [group][64-column chunk of P]: written by the group
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ constexpr int round16(int x) { return (x + 15) & ~15; }

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// One arrival per warp on a barrier that counts warps: every lane's earlier
// tcgen05 and shared-memory accesses are ordered before the warp-wide sync,
// after which lane 0 arrives (a warp-collective call; the warp must be
// converged).  One shared-memory atomic per warp instead of 32.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Agent set coordinates (h, b) of slice bh for the 4-D agents tensor map.
__device__ __forceinline__ void agent_coords(long long bh, int H, int b_sets, int* h, int* b) {
  *h = (int)(bh % H);
  *b = b_sets > 1 ? (int)(bh / H) : 0;
}

// Bounded wait for an issuer's last commit before TMEM is released.
__device__ __forceinline__ void drain_commits(uint64_t* bar) {
  mma_commit(bar);
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, 0) && globaltimer() - t0 < kWaitLimitNs) {
  }
}

// ============================================================== aggregation
// The two fp16 logits of a bias word as floats.
__device__ __forceinline__ float2 bias_pair(uint32_t w) {
  __half2 h;
  memcpy(&h, &w, sizeof(h));
  return __half22float2(h);
}

constexpr size_t kAggSmemBytes = 1024 + 2 * (size_t)kAgentBufBytes +
                                 2 * (size_t)kAggStages * kKTileBytes + sizeof(AggBars);

// kBias: the agent bias B1 is added to the score tiles (a separate
// instantiation, so the unbiased kernel carries none of its code).
template <bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
    agent_aggregate_tc_kernel(const __grid_constant__ CUtensorMap map_k,
                              const __grid_constant__ CUtensorMap map_v,
                              const __grid_constant__ CUtensorMap map_a, int a_sets,
                              AggParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;                                  // 2 agent tile buffers
  uint8_t* sK = sA + 2 * kAgentBufBytes;
  uint8_t* sV = sK + kAggStages * kKTileBytes;
  AggBars* bars = reinterpret_cast<AggBars*>(sV + kAggStages * kKTileBytes);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long cta = blockIdx.x;
  const long long t_begin = (cta * p.total_tiles) / p.ctas;
  const long long t_end = ((cta + 1) * p.total_tiles) / p.ctas;
  const int tps = p.tiles_per_slice;
  const bool two = p.k > 128;                 // two 128-row agent tiles
  const int d16 = (p.d + 15) >> 4;            // K steps of S = A K^T
  const int dn = d16 * 16;                    // N of U += P V

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAggStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], two ? 2 : 1);   // released by every group that used the tile
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->a_full[b], 1);
      mbar_init(&bars->a_empty[b], 2);            // both issuers finish the segment
    }
    for (int g = 0; g < 2; ++g) {
      for (int b = 0; b < kSBuf; ++b) {
        mbar_init(&bars->s_full[g][b], 1);
        mbar_init(&bars->p_full[g][b], kSoftmaxWarps);
        mbar_init(&bars->pv_done[g][b], 1);
      }
      mbar_init(&bars->drain[g], 1);
    }
    mbar_init(&bars->x_pub, kSoftmaxWarps);
    mbar_init(&bars->x_done, kSoftmaxWarps);
    bars->abort = 0;
    mbar_fence_init();
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_a);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  constexpr bool biased = kBias;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = bars->tmem_base;
  // TMEM columns of group g: score buffers at g*256 + {0, 64, 128} (the bf16
  // P of a tile is written over the first 32 columns of its scores), U at
  // g*256 + 192 (dn <= 64).  A score buffer is free again once the P V that
  // read its P has completed.

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      long long it = 0;
      int seg = 0, a_loads = 0;
      const uint32_t a_bytes = (two ? 256 : 128) * kRowBytes;
      pdl_wait();             // the agents may come from the previous kernel
      for (long long t = t_begin; t < t_end; ++seg) {
        const long long bh = t / tps;
        const long long seg_end = min(t_end, (bh + 1) * tps);
        // the segment's agents go to buffer seg % 2 once segment seg - 2 is
        // done with it, so they load while segment seg - 1 still computes
        const int ab = seg & 1;
        if (seg >= 2 && !mbar_wait(&bars->a_empty[ab], (uint32_t)((seg - 2) >> 1) & 1, abort))
          break;
        int h, b;
        agent_coords(bh, p.H, a_sets, &h, &b);
        mbar_expect_tx(&bars->a_full[ab], a_bytes);
        tma_load_4d(sA + ab * kAgentBufBytes, &map_a, &bars->a_full[ab], 0, 0, h, b);
        ++a_loads;
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
      // On abort, wait (bounded) for the loads already issued before leaving:
      // the key tiles still in the ring and the last two agent tiles.
      if (*abort) {
        for (long long j = (it > kAggStages ? it - kAggStages : 0); j < it; ++j) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars->full[j % kAggStages], (uint32_t)(j / kAggStages) & 1) &&
                 globaltimer() - t0 < kWaitLimitNs) {
          }
        }
        for (int sg = (a_loads > 2 ? a_loads - 2 : 0); sg < a_loads; ++sg) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars->a_full[sg & 1], (uint32_t)(sg >> 1) & 1) &&
                 globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp < kFirstSoftmaxWarp) {
    if (lane == 0) {
      // ------------------------------------- MMA issuer of group g = warp - 1
      const int g = warp - 1;
      const uint32_t idesc_s = idesc_bf16(128, kKeyTile, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, dn, 0, 1);
      const uint32_t sA_half = smem_u32(sA) + (two ? g : 0) * 128 * kRowBytes;
      const uint32_t sK_addr = smem_u32(sK), sV_addr = smem_u32(sV);
      const uint32_t u_tm = tmem + g * 256 + 192;
      long long it0 = 0;
      int seg = 0;
      int cnt_s = 0, cnt_p = 0;
      bool ok = true;
      for (long long t = t_begin; t < t_end && ok; ++seg) {
        const long long bh = t / tps;
        const long long seg_end = min(t_end, (bh + 1) * tps);
        const int n = (int)(seg_end - t);
        const int ab = seg & 1;
        const uint32_t sA_addr = sA_half + ab * kAgentBufBytes;
        if (!mbar_wait(&bars->a_full[ab], (uint32_t)(seg >> 1) & 1, abort)) break;
        tc_fence_after();
        bool first = true;
        auto issue_s = [&](int i) -> bool {
          const long long itg = it0 + i;
          const int s = (int)(itg % kAggStages);
          if (!mbar_wait(&bars->full[s], (uint32_t)(itg / kAggStages) & 1, abort)) return false;
          const int J = cnt_s, b = J % kSBuf;
          if (J >= kSBuf &&
              !mbar_wait(&bars->pv_done[g][b], (uint32_t)(J / kSBuf - 1) & 1, abort))
            return false;           // the buffer's previous P has been consumed
          tc_fence_after();
          const uint32_t d_tm = tmem + g * 256 + b * 64;
          for (int kk = 0; kk < d16; ++kk) {
            const uint64_t da = sw128_desc(sA_addr + kk * 32, 16);
            const uint64_t db = sw128_desc(sK_addr + s * kKTileBytes + kk * 32, 16);
            mma_ss(d_tm, da, db, idesc_s, kk > 0);
          }
          mma_commit(&bars->s_full[g][b]);
          ++cnt_s;
          return true;
        };
        auto issue_pv = [&](int i) -> bool {
          const long long itg = it0 + i;
          const int s = (int)(itg % kAggStages);
          const int J = cnt_p, b = J % kSBuf;
          if (!mbar_wait(&bars->p_full[g][b], (uint32_t)(J / kSBuf) & 1, abort)) return false;
          tc_fence_after();
          const uint32_t p_tm = tmem + g * 256 + b * 64;
          for (int kk = 0; kk < kKeyTile / 16; ++kk) {
            const uint64_t dv = sw128_desc(sV_addr + s * kKTileBytes + kk * 2048, 8192);
            mma_ts(u_tm, p_tm + kk * 8, dv, idesc_pv, (!first || kk > 0) ? 1u : 0u);
          }
          first = false;
          mma_commit(&bars->pv_done[g][b]);
          mma_commit(&bars->empty[s]);
          ++cnt_p;
          return true;
        };
        // this group's tiles of the segment: all of them for two agent tiles,
        // else every other one; two tiles of look-ahead (S of the tile after
        // next is issued before P V of the current one, into the buffer whose
        // P V has completed)
        const int i0 = two ? 0 : g, step = two ? 1 : 2;
        // In two-agent-tile mode both groups take every key tile; start group 1
        // one softmax behind group 0 so their SFU-bound phases interleave.
        if (two && g == 1 && seg == 0 && n > 0 &&
            !mbar_wait(&bars->p_full[0][0], 0, abort))
          ok = false;
        constexpr int kAhead = kSBuf - 1;
        for (int q = 0, i = i0; q < kAhead && i < n && ok; ++q, i += step) ok = issue_s(i);
        for (int i = i0; i < n && ok; i += step) {
          if (i + kAhead * step < n) ok = issue_s(i + kAhead * step);
          if (ok) ok = issue_pv(i);
        }
        mma_commit(&bars->a_empty[ab]);
        it0 += n;
        t = seg_end;
      }
      drain_commits(&bars->drain[g]);
    }
  } else {
    // ---------------------------------------------------- softmax groups
    // Every thread walks the same segments and tiles whatever happens; after a
    // failed (timed-out) wait it only skips work, so no barrier is left short.
    // A warp owns a 16-row slab of its group's 128 TMEM lanes with all 64
    // columns of each score tile: the 4 threads of a row reduce its maximum
    // and sum with shuffles, so the warps of a group never wait for each other
    // inside a tile.
    const int sw = warp - kFirstSoftmaxWarp;  // 0..15
    const int g = sw >> 3;                    // group 0: warps 3-10, group 1: warps 11-18
    const int quad = warp & 3;                // TMEM lane quadrant this warp may access
    const int slab = quad * 32 + ((sw >> 2) & 1) * 16;   // first lane (row) of the slab
    const int j4 = lane & 3;
    const int r0 = slab + (lane >> 2), r1 = r0 + 8;      // this thread's two rows
    const uint32_t slab_off = (uint32_t)slab << 16;
    const uint32_t u_col = tmem + slab_off + g * 256 + 192;
    const int row_base = two ? g * 128 : 0;   // agent of TMEM lane 0 in this group
    const bool warp_active = row_base + slab < p.k;
    int J = 0, seg = 0;
    bool ok = true;
    for (long long t = t_begin; t < t_end; ++seg) {
      const long long bh = t / tps;
      const long long seg_end = min(t_end, (bh + 1) * tps);
      const int n = (int)(seg_end - t);
      const int n_mine = two ? n : (g == 0 ? (n + 1) / 2 : n / 2);
      // running maxima (log2 units) and this thread's partial sums of its rows
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      bool first = true;
      for (int i = 0; i < n; ++i) {
        if (!two && (i & 1) != g) continue;
        const int b = J % kSBuf;
        const uint32_t s_col = tmem + slab_off + g * 256 + b * 64;
        const int valid = min(kKeyTile, p.N - (int)(t + i - bh * tps) * kKeyTile);
        // the tile's B1 logits of this thread's column pairs (two fp16 per
        // word), loaded before the wait for the scores so that their latency
        // overlaps it; columns past the slice (and padding agents) add 0
        uint32_t bw0[8], bw1[8];
        if constexpr (kBias) {
          const int n0 = (int)(t + i - bh * tps) * kKeyTile;
          const long long ra0 = (long long)(bh % p.H) * p.k + row_base + r0;
          const bool in0 = ok && row_base + r0 < p.k, in1 = ok && row_base + r1 < p.k;
          const uint32_t* w0p =
              reinterpret_cast<const uint32_t*>(p.bias.dense + ra0 * p.bias.ld + n0);
          const uint32_t* w1p = w0p + 4LL * p.bias.ld;     // 8 agent rows further
#pragma unroll
          for (int g8 = 0; g8 < 8; ++g8) {
            const int col = 8 * g8 + 2 * j4;
            bw0[g8] = (in0 && col < valid) ? __ldg(w0p + col / 2) : 0u;
            bw1[g8] = (in1 && col < valid) ? __ldg(w1p + col / 2) : 0u;
          }
        }
        if (ok) ok = warp_wait(&bars->s_full[g][b], (uint32_t)(J / kSBuf) & 1, abort);
        tc_fence_after();
        // A tile's scores are only written after the P V of the buffer's
        // previous tile (which needed every warp's P) has completed, so the
        // warps of a group are never more than kSBuf - 1 tiles apart and a
        // barrier phase only ever collects arrivals of one tile.
        if (ok && warp_active) {
          float v[32];
          slab_ld64(s_col, v);
          if (valid < kKeyTile) slab_mask<8>(v, 0, j4, valid);   // ragged last tile
          if (biased) {
            // scores become log2-unit logits S*c + B1*log2(e), then ce = 1
#pragma unroll
            for (int g8 = 0; g8 < 8; ++g8) {
              const float2 b0 = bias_pair(bw0[g8]), b1 = bias_pair(bw1[g8]);
              v[4 * g8] = fmaf(v[4 * g8], p.c, b0.x);
              v[4 * g8 + 1] = fmaf(v[4 * g8 + 1], p.c, b0.y);
              v[4 * g8 + 2] = fmaf(v[4 * g8 + 2], p.c, b1.x);
              v[4 * g8 + 3] = fmaf(v[4 * g8 + 3], p.c, b1.y);
            }
          }
          const float ce = biased ? 1.f : p.c;
          float t0 = -INFINITY, t1 = -INFINITY;
          slab_max<8>(v, t0, t1);
          t0 = row4_max(t0) * ce;
          t1 = row4_max(t1) * ce;
          if (first) {
            m0 = t0;
            m1 = t1;
            first = false;
          } else if (__any_sync(0xffffffffu,
                                t0 > m0 + kRescaleThreshold || t1 > m1 + kRescaleThreshold)) {
            // a running max grew a lot: once the previous P V has landed,
            // rescale the slab's U rows and sums by 2^(m_old - m_new)
            ok = warp_wait(&bars->pv_done[g][(J - 1) % kSBuf], (uint32_t)((J - 1) / kSBuf) & 1,
                           abort);
            tc_fence_after();
            if (ok) {
              const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
              const float a0 = ex2(m0 - n0), a1 = ex2(m1 - n1);
              m0 = n0;
              m1 = n1;
              l0 *= a0;
              l1 *= a1;
#pragma unroll 1
              for (int c = 0; c < dn; c += 16) {
                float u[8];
                slab_ld16(u_col + c, u);
                u[0] *= a0; u[1] *= a0; u[2] *= a1; u[3] *= a1;
                u[4] *= a0; u[5] *= a0; u[6] *= a1; u[7] *= a1;
                slab_st16(u_col + c, u);
              }
            }
          }
          if (ok) {
            uint32_t pk[16];
            slab_exp<8>(v, ce, -m0, -m1, pk, l0, l1);
            slab_st_p32(s_col, pk);
            tmem_wait_st();
          }
        }
        warp_arrive(&bars->p_full[g][b]);
        ++J;
      }
      // ---- segment epilogue: write this CTA's partial for slice bh
      const int slot = (int)(cta - ((bh * tps + 1) * p.ctas - 1) / p.total_tiles);
      const long long slot_row = (bh * p.slots + slot) * (long long)p.k;
      if (n_mine > 0 && ok)
        ok = warp_wait(&bars->pv_done[g][(J - 1) % kSBuf], (uint32_t)((J - 1) / kSBuf) & 1,
                       abort);
      tc_fence_after();
      l0 = row4_sum(l0);
      l1 = row4_sum(l1);
      if (two) {
        if (ok && warp_active) {            // warp-uniform: the TMEM loads are warp-collective
          const int a0 = row_base + r0, a1 = row_base + r1;
#pragma unroll 1
          for (int c = 0; c < dn; c += 16) {
            float u[8];
            slab_ld16(u_col + c, u);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int col = c + 8 * h + 2 * j4;
              if (c + 8 * h < p.d) {
                if (a0 < p.k)
                  *reinterpret_cast<float2*>(p.part_u + (slot_row + a0) * p.d + col) =
                      make_float2(u[4 * h], u[4 * h + 1]);
                if (a1 < p.k)
                  *reinterpret_cast<float2*>(p.part_u + (slot_row + a1) * p.d + col) =
                      make_float2(u[4 * h + 2], u[4 * h + 3]);
              }
            }
          }
          if (j4 == 0) {
            if (a0 < p.k)
              *reinterpret_cast<float2*>(p.part_ml + (slot_row + a0) * 2) = make_float2(m0, l0);
            if (a1 < p.k)
              *reinterpret_cast<float2*>(p.part_ml + (slot_row + a1) * 2) = make_float2(m1, l1);
          }
        }
      } else if (g == 1) {
        // both groups hold the same agent rows over different key tiles:
        // group 1 publishes (m, l) and waits until group 0 has read its
        // accumulators
        if (j4 == 0) {
          bars->m_x[r0] = m0;
          bars->m_x[r1] = m1;
          bars->l_x[r0] = l0;
          bars->l_x[r1] = l1;
        }
        warp_arrive(&bars->x_pub);
        if (ok) ok = warp_wait(&bars->x_done, (uint32_t)seg & 1, abort);
        tc_fence_after();
      } else {
        if (ok) ok = warp_wait(&bars->x_pub, (uint32_t)seg & 1, abort);
        tc_fence_after();
        if (ok && warp_active) {            // warp-uniform: the TMEM loads are warp-collective
          const bool has1 = (n / 2) > 0;
          const uint32_t u1_col = tmem + slab_off + 256 + 192;
          float mm0 = m0, mm1 = m1, s0 = 1.f, s1 = 1.f, w0 = 0.f, w1 = 0.f;
          if (has1) {
            const float x0 = bars->m_x[r0], x1 = bars->m_x[r1];
            mm0 = fmaxf(m0, x0);
            mm1 = fmaxf(m1, x1);
            s0 = ex2(m0 - mm0);
            s1 = ex2(m1 - mm1);
            w0 = ex2(x0 - mm0);
            w1 = ex2(x1 - mm1);
          }
#pragma unroll 1
          for (int c = 0; c < dn; c += 16) {
            float u[8];
            slab_ld16(u_col + c, u);
            if (has1) {
              float w[8];
              slab_ld16(u1_col + c, w);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                u[4 * h] = s0 * u[4 * h] + w0 * w[4 * h];
                u[4 * h + 1] = s0 * u[4 * h + 1] + w0 * w[4 * h + 1];
                u[4 * h + 2] = s1 * u[4 * h + 2] + w1 * w[4 * h + 2];
                u[4 * h + 3] = s1 * u[4 * h + 3] + w1 * w[4 * h + 3];
              }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int col = c + 8 * h + 2 * j4;
              if (c + 8 * h < p.d) {
                if (r0 < p.k)
                  *reinterpret_cast<float2*>(p.part_u + (slot_row + r0) * p.d + col) =
                      make_float2(u[4 * h], u[4 * h + 1]);
                if (r1 < p.k)
                  *reinterpret_cast<float2*>(p.part_u + (slot_row + r1) * p.d + col) =
                      make_float2(u[4 * h + 2], u[4 * h + 3]);
              }
            }
          }
          if (j4 == 0) {
            const float lt0 = s0 * l0 + (has1 ? w0 * bars->l_x[r0] : 0.f);
            const float lt1 = s1 * l1 + (has1 ? w1 * bars->l_x[r1] : 0.f);
            if (r0 < p.k)
              *reinterpret_cast<float2*>(p.part_ml + (slot_row + r0) * 2) = make_float2(mm0, lt0);
            if (r1 < p.k)
              *reinterpret_cast<float2*>(p.part_ml + (slot_row + r1) * 2) = make_float2(mm1, lt1);
          }
        }
        warp_arrive(&bars->x_done);
      }
      // group 1 writes m_x / l_x again only after the next segment's x_done
      // phase, which follows group 0's reads of this one
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
                                sizeof(BcBars);

// Row maxima of a slab's two rows (this thread's columns) over score columns
// [0, kpad), columns >= k masked; 64 columns per TMEM load, then 32 and 16.
__device__ __forceinline__ void bc_slab_max(uint32_t s_col, int k, int kpad, int j4, float& t0,
                                            float& t1) {
  int c = 0;
#pragma unroll 1
  for (; c + 64 <= kpad; c += 64) {
    float v[32];
    slab_ld64(s_col + c, v);
    if (c + 64 > k) slab_mask<8>(v, c, j4, k);
    slab_max<8>(v, t0, t1);
  }
  if (c + 32 <= kpad) {
    float v[16];
    slab_ld32(s_col + c, v);
    if (c + 32 > k) slab_mask<4>(v, c, j4, k);
    slab_max<4>(v, t0, t1);
    c += 32;
  }
  if (c < kpad) {
    float v[8];
    slab_ld16(s_col + c, v);
    if (c + 16 > k) slab_mask<2>(v, c, j4, k);
    slab_max<2>(v, t0, t1);
  }
}

// The B2 logits of a slab's two query rows: the rows of the dense copy as
// 32-bit words (two fp16 agents each), null for a row past the slice.
struct BcRowBias {
  const uint32_t* w0;
  const uint32_t* w1;
};

// The words of a 16x256b register block (first column c): agents
// c + 8 g + 2 j4 and the next one.
template <int R>
__device__ __forceinline__ void bc_bias_load(uint32_t (&w0)[R], uint32_t (&w1)[R], int c, int j4,
                                             const BcRowBias& rb) {
#pragma unroll
  for (int g = 0; g < R; ++g) {
    const int w = (c + 8 * g) / 2 + j4;
    w0[g] = rb.w0 ? __ldg(rb.w0 + w) : 0u;
    w1[g] = rb.w1 ? __ldg(rb.w1 + w) : 0u;
  }
}
// Scores of the block become log2-unit logits S*c + B2*log2(e); masked
// columns stay -inf (their bias words are the zero padding).
template <int R>
__device__ __forceinline__ void bc_bias_add(float (&v)[4 * R], const uint32_t (&w0)[R],
                                            const uint32_t (&w1)[R], float cs) {
#pragma unroll
  for (int g = 0; g < R; ++g) {
    const float2 b0 = bias_pair(w0[g]), b1 = bias_pair(w1[g]);
    v[4 * g] = fmaf(v[4 * g], cs, b0.x);
    v[4 * g + 1] = fmaf(v[4 * g + 1], cs, b0.y);
    v[4 * g + 2] = fmaf(v[4 * g + 2], cs, b1.x);
    v[4 * g + 3] = fmaf(v[4 * g + 3], cs, b1.y);
  }
}

// Biased max pass: adds B2 to every score, writes the logits back over the
// scores (the exponential pass then uses scale 1) and returns the row maxima.
// w0, w1 hold the first 64-column block's bias words (loaded by the caller
// before it waited for the scores, when kpad >= 64); each later block's words
// are requested as soon as the previous block has used its own.
__device__ __forceinline__ void bc_slab_bias_max(uint32_t s_col, int k, int kpad, int j4,
                                                 float cs, const BcRowBias& rb, float& t0,
                                                 float& t1, uint32_t (&w0)[8],
                                                 uint32_t (&w1)[8]) {
  int c = 0;
#pragma unroll 1
  for (; c + 64 <= kpad; c += 64) {
    float v[32];
    slab_ld64(s_col + c, v);
    if (c + 64 > k) slab_mask<8>(v, c, j4, k);
    bc_bias_add<8>(v, w0, w1, cs);
    if (c + 128 <= kpad) bc_bias_load<8>(w0, w1, c + 64, j4, rb);
    slab_st64(s_col + c, v);
    slab_max<8>(v, t0, t1);
  }
  if (c + 32 <= kpad) {
    uint32_t u0[4], u1[4];
    bc_bias_load<4>(u0, u1, c, j4, rb);
    float v[16];
    slab_ld32(s_col + c, v);
    if (c + 32 > k) slab_mask<4>(v, c, j4, k);
    bc_bias_add<4>(v, u0, u1, cs);
    slab_st32(s_col + c, v);
    slab_max<4>(v, t0, t1);
    c += 32;
  }
  if (c < kpad) {
    uint32_t u0[2], u1[2];
    bc_bias_load<2>(u0, u1, c, j4, rb);
    float v[8];
    slab_ld16(s_col + c, v);
    if (c + 16 > k) slab_mask<2>(v, c, j4, k);
    bc_bias_add<2>(v, u0, u1, cs);
    slab_st16(s_col + c, v);
    slab_max<2>(v, t0, t1);
  }
  tmem_wait_st();
}

// TMEM column (within a 256-column buffer) of the bf16 P of 64-score-column
// chunk ch.  "Packed" layout (S and O fit side by side, kpad + dn <= 256):
// chunk ch's P at 32 ch, i.e. each score column's P at half its column, and
// O at kpad.  "Wide" layout (kpad + dn > 256): chunks 0 and 1 pack into
// [0, 64), O takes [64, 128) once chunk 1 has been read, and every later
// chunk's P stays at the start of its own score columns.  Either way a P
// store only lands on score columns its warp has already read and never on
// O, so P V can run while later chunks are still being computed.
__device__ __forceinline__ int bc_p_col(int ch, bool wide) { return (wide && ch >= 2) ? 64 * ch : 32 * ch; }

// P = 2^(S*c - m_row) as bf16 for score columns [0, kpad) (columns >= k give
// 0), placed by bc_p_col.  Adds the exponentials to the partial row sums l0,
// l1.  After each 64-column chunk the warp arrives on that chunk's barrier
// (whether or not it did the work).
// kStoreP: the packed bf16 P words of the thread's two rows also go to global
// memory, rows g0 and g1 (bf16x2 words of a [kpad]-wide row; null: the row
// is past the slice), for the backward pass's query gradient kernel.
template <int R, bool kStoreP>
__device__ __forceinline__ void bc_store_p(uint32_t* g0, uint32_t* g1, int c, int j4,
                                           const uint32_t (&pk)[2 * R]) {
  if constexpr (kStoreP) {
#pragma unroll
    for (int g = 0; g < R; ++g) {
      if (g0) g0[(c + 8 * g) / 2 + j4] = pk[2 * g];
      if (g1) g1[(c + 8 * g) / 2 + j4] = pk[2 * g + 1];
    }
  }
}

// Column mode (colm non-null, kStoreP): the exponent subtracts the column's
// max colm[2 a] (log2 units) instead of the row's: v = S*c_scale - m_a.
template <int R>
__device__ __forceinline__ void bc_col_shift(float (&v)[4 * R], int c, int j4, int k,
                                             float c_scale, const float* colm) {
#pragma unroll
  for (int g = 0; g < R; ++g) {
    const int a = c + 8 * g + 2 * j4;
    const float m0 = a < k ? __ldg(colm + 2 * a) : 0.f;
    const float m1 = a + 1 < k ? __ldg(colm + 2 * a + 2) : 0.f;
    v[4 * g] = fmaf(v[4 * g], c_scale, -m0);
    v[4 * g + 1] = fmaf(v[4 * g + 1], c_scale, -m1);
    v[4 * g + 2] = fmaf(v[4 * g + 2], c_scale, -m0);
    v[4 * g + 3] = fmaf(v[4 * g + 3], c_scale, -m1);
  }
}

template <bool kStoreP = false>
__device__ __forceinline__ void bc_slab_exp(uint32_t s_col, int k, int kpad, int j4, bool wide,
                                            float c_scale, float neg_m0, float neg_m1, float& l0,
                                            float& l1, bool run, uint64_t* chunk_bar,
                                            uint32_t* g0 = nullptr, uint32_t* g1 = nullptr,
                                            const float* colm = nullptr) {
  const bool col_mode = kStoreP && colm != nullptr;
  const float cs_col = c_scale;            // column mode: S*c - m_a, then exp2 as is
  if (col_mode) {
    c_scale = 1.f;
    neg_m0 = neg_m1 = 0.f;
  }
  int c = 0, ch = 0;
#pragma unroll 1
  for (; c + 64 <= kpad; c += 64, ++ch) {
    if (run) {
      float v[32];
      uint32_t pk[16];
      slab_ld64(s_col + c, v);
      if (c + 64 > k) slab_mask<8>(v, c, j4, k);
      if (col_mode) bc_col_shift<8>(v, c, j4, k, cs_col, colm);
      slab_exp<8>(v, c_scale, neg_m0, neg_m1, pk, l0, l1);
      slab_st_p32(s_col + bc_p_col(ch, wide), pk);
      bc_store_p<8, kStoreP>(g0, g1, c, j4, pk);
      tmem_wait_st();
    }
    warp_arrive(&chunk_bar[ch]);
  }
  if (c < kpad) {
    if (run) {
      const uint32_t pc = s_col + bc_p_col(ch, wide);
      if (c + 32 <= kpad) {
        float v[16];
        uint32_t pk[8];
        slab_ld32(s_col + c, v);
        if (c + 32 > k) slab_mask<4>(v, c, j4, k);
        if (col_mode) bc_col_shift<4>(v, c, j4, k, cs_col, colm);
        slab_exp<4>(v, c_scale, neg_m0, neg_m1, pk, l0, l1);
        slab_st_p16(pc, pk);
        bc_store_p<4, kStoreP>(g0, g1, c, j4, pk);
      }
      const int c16 = c + ((kpad - c) & 32);
      if (c16 < kpad) {
        float v[8];
        uint32_t pk[4];
        slab_ld16(s_col + c16, v);
        if (c16 + 16 > k) slab_mask<2>(v, c16, j4, k);
        if (col_mode) bc_col_shift<2>(v, c16, j4, k, cs_col, colm);
        slab_exp<2>(v, c_scale, neg_m0, neg_m1, pk, l0, l1);
        slab_st_p8(pc + (c16 - c) / 2, pk);
        bc_store_p<2, kStoreP>(g0, g1, c16, j4, pk);
      }
      tmem_wait_st();
    }
    warp_arrive(&chunk_bar[ch]);
  }
}

// kBias: the agent bias B2 is added in the max pass; kStats: the epilogue
// writes the backward pass's per-query statistics (p.stats) instead of O
// (separate instantiations).
template <bool kBias, bool kStats = false>
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
  BcBars* bars = reinterpret_cast<BcBars*>(sO + 2 * kQTileBytes);
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
  // Columns of a 256-column TMEM buffer: S over [0, kpad); P and O placed as
  // bc_p_col describes.
  const bool wide = kpad + dn > 256;
  const int o_col = wide ? 64 : kpad;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBcStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    mbar_init(&bars->ag_full, 1);
    mbar_init(&bars->ag_empty, 2);          // both issuers are done with the slice
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      for (int c = 0; c < 4; ++c) mbar_init(&bars->p_chunk[i][c], kSoftmaxWarps);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_free[i], kSoftmaxWarps);
      mbar_init(&bars->drain[i], 1);
    }
    bars->abort = 0;
    mbar_fence_init();
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_va);
    prefetch_tensormap(&map_o);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = bars->tmem_base;
  // TMEM: buffer g (tiles j with j % 2 == g) at column g*256 holds S, then P
  // and O as laid out above.

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      long long cur = -1;
      int n_slices = 0;
      const uint32_t ag_bytes = 2u * kpad * kRowBytes;
      pdl_wait();             // agents and V_A come from the previous kernels
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
  } else if (warp < kFirstSoftmaxWarp) {
    if (lane == 0) {
      // ----------------------------- MMA issuer of group g (tiles j % 2 == g)
      const int g = warp - 1;
      const uint32_t idesc_s = idesc_bf16(128, kpad, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, dn, 0, 1);
      const uint32_t sA_addr = smem_u32(sA), sVA_addr = smem_u32(sVA), sQ_addr = smem_u32(sQ);
      const uint32_t s_tm = tmem + g * 256;
      const uint32_t o_tm = s_tm + o_col;
      int n_slices = 0, u = 0;
      long long cur = -1;
      bool ok = true;
      // walk every tile so that slice boundaries are seen by both issuers
      for (int j = 0; j < n_tiles && ok; ++j) {
        const long long bh = (t_begin + j) / tps;
        if (bh != cur) {
          if (cur >= 0) mma_commit(&bars->ag_empty);   // done with the previous slice
          if (!mbar_wait(&bars->ag_full, n_slices & 1, abort)) {
            ok = false;
            break;
          }
          cur = bh;
          ++n_slices;
        }
        if ((j & 1) != g) continue;
        const int s = j % kBcStages;
        // Start group 1 one softmax behind group 0, so that one group's
        // exponentials overlap the other group's MMA and epilogue phases
        // instead of both contending for the SFU at the same time.
        if (g == 1 && u == 0 && !mbar_wait(&bars->p_chunk[0][(kpad - 1) / 64], 0, abort)) {
          ok = false;
          break;
        }
        // S = Q A^T into this group's buffer once its previous O has been read
        if (u >= 1 && !mbar_wait(&bars->o_free[g], (u - 1) & 1, abort)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&bars->q_full[s], (j / kBcStages) & 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kk = 0; kk < d16; ++kk) {
          const uint64_t da = sw128_desc(sQ_addr + s * kQTileBytes + kk * 32, 16);
          const uint64_t db = sw128_desc(sA_addr + kk * 32, 16);
          mma_ss(s_tm, da, db, idesc_s, kk > 0);
        }
        mma_commit(&bars->s_full[g]);
        mma_commit(&bars->q_empty[s]);
        // O = P V_A, 64 agents at a time as the group writes P (in the wide
        // layout O's columns are free only once chunk 1 has been read)
        int kk = 0;
        for (int ch = 0; ch * 64 < kpad && ok; ++ch) {
          if (!mbar_wait(&bars->p_chunk[g][ch], u & 1, abort)) {
            ok = false;
            break;
          }
          if (wide && ch == 0) continue;
          tc_fence_after();
          const int kk_end = min(kpad / 16, 4 * ch + 4);
          for (; kk < kk_end; ++kk)   // agents [16 kk, 16 kk + 16)
            mma_ts(o_tm, s_tm + bc_p_col(kk >> 2, wide) + (kk & 3) * 8,
                   sw128_desc(sVA_addr + kk * 2048, 8192), idesc_pv, kk > 0);
        }
        if (!ok) break;
        mma_commit(&bars->o_full[g]);
        ++u;
      }
      if (ok && cur >= 0) mma_commit(&bars->ag_empty);
      drain_commits(&bars->drain[g]);
    }
  } else {
    // ------------------------------------------- softmax + epilogue groups
    // A warp owns a 16-row slab of the group's 128 query rows with all k
    // score columns; the 4 threads of a row reduce its maximum and sum with
    // shuffles, so within a tile the warps only meet at the output staging.
    const int sw = warp - kFirstSoftmaxWarp;
    const int g = sw >> 3;
    const int quad = warp & 3;
    const int slab = quad * 32 + ((sw >> 2) & 1) * 16;
    const int j4 = lane & 3;
    const int r0 = slab + (lane >> 2), r1 = r0 + 8;
    const uint32_t s_col = tmem + ((uint32_t)slab << 16) + g * 256;
    const uint32_t o_tm = s_col + o_col;
    uint8_t* stage = sO + g * kQTileBytes;
    const bool leader = (warp == kFirstSoftmaxWarp + 8 * g) && lane == 0;
    const int n_ch = dn / 16;                // 16-column chunks of O
    bool ok = true;
    for (int j = g; j < n_tiles; j += 2) {
      const int u = j >> 1;
      const long long t = t_begin + j;
      const long long bh = t / tps;
      const int q0 = (int)(t - bh * tps) * kQTile;
      // biased: the rows' B2 words of the first 64 agents are requested
      // before the wait, so that their latency overlaps it
      BcRowBias rb;
      uint32_t bw0[8], bw1[8];
      if constexpr (kBias) {
        const __half* hb = p.bias.dense + (long long)(bh % p.H) * p.N * p.bias.ld;
        rb.w0 = q0 + r0 < p.N
                    ? reinterpret_cast<const uint32_t*>(hb + (long long)(q0 + r0) * p.bias.ld)
                    : nullptr;
        rb.w1 = q0 + r1 < p.N
                    ? reinterpret_cast<const uint32_t*>(hb + (long long)(q0 + r1) * p.bias.ld)
                    : nullptr;
        if (kpad >= 64) bc_bias_load<8>(bw0, bw1, 0, j4, rb);
      }
      if (ok) ok = warp_wait(&bars->s_full[g], u & 1, abort);
      tc_fence_after();
      float l0 = 0.f, l1 = 0.f, t0 = -INFINITY, t1 = -INFINITY;
      const float ce = kBias ? 1.f : p.c;     // biased scores are already logits
      if (ok) {
        if constexpr (kBias) {
          bc_slab_bias_max(s_col, p.k, kpad, j4, p.c, rb, t0, t1, bw0, bw1);
        } else if (!(kStats && p.stats.col_ml)) {   // column mode: no row max
          bc_slab_max(s_col, p.k, kpad, j4, t0, t1);
        }
        t0 = row4_max(t0) * ce;
        t1 = row4_max(t1) * ce;
      }
      if constexpr (kStats) {
        uint32_t* g0 = q0 + r0 < p.N ? reinterpret_cast<uint32_t*>(
                                           p.stats.p + (bh * p.N + q0 + r0) * (long long)kpad)
                                     : nullptr;
        uint32_t* g1 = q0 + r1 < p.N ? reinterpret_cast<uint32_t*>(
                                           p.stats.p + (bh * p.N + q0 + r1) * (long long)kpad)
                                     : nullptr;
        const float* colm = p.stats.col_ml ? p.stats.col_ml + bh * p.k * 2 : nullptr;
        bc_slab_exp<true>(s_col, p.k, kpad, j4, wide, ce, -t0, -t1, l0, l1, ok, bars->p_chunk[g],
                          g0, g1, colm);
      } else {
        bc_slab_exp(s_col, p.k, kpad, j4, wide, ce, -t0, -t1, l0, l1, ok, bars->p_chunk[g]);
      }
      const float sum0 = row4_sum(l0), sum1 = row4_sum(l1);
      const float inv0 = 1.f / sum0, inv1 = 1.f / sum1;
      // epilogue: O = (P V_A) / l -> bf16 -> swizzled staging tile -> TMA store
      if (ok) ok = warp_wait(&bars->o_full[g], u & 1, abort);
      tc_fence_after();
      float o[4][8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (ok && q < n_ch) {
          slab_ld16(o_tm + q * 16, o[q]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[q][e] = 0.f;
        }
      }
      warp_arrive(&bars->o_free[g]);           // the buffer may take the next S now
      if constexpr (kStats) {
        if (p.stats.col_ml) continue;          // column mode: the exponentials only
        // D = dO . O over the row's columns (this thread's pairs, then the 4
        // threads of the row), and the row's max and sum, by its first thread
        const bool in0 = q0 + r0 < p.N, in1 = q0 + r1 < p.N;
        const long long row0 = bh * p.N + q0 + r0, row1 = row0 + 8;
        const __nv_bfloat16* g0 = p.stats.dout + row0 * p.d + 2 * j4;
        const __nv_bfloat16* g1 = p.stats.dout + row1 * p.d + 2 * j4;
        float dd0 = 0.f, dd1 = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ch = 2 * q + h;
            if (ch * 8 < p.d) {
              if (in0) {
                const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(g0 + ch * 8));
                dd0 = fmaf(bf16x2_lo(w), o[q][4 * h] * inv0, dd0);
                dd0 = fmaf(bf16x2_hi(w), o[q][4 * h + 1] * inv0, dd0);
              }
              if (in1) {
                const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(g1 + ch * 8));
                dd1 = fmaf(bf16x2_lo(w), o[q][4 * h + 2] * inv1, dd1);
                dd1 = fmaf(bf16x2_hi(w), o[q][4 * h + 3] * inv1, dd1);
              }
            }
          }
        }
        dd0 = row4_sum(dd0);
        dd1 = row4_sum(dd1);
        if (ok && j4 == 0) {
          if (in0) {
            p.stats.m[row0] = t0;
            p.stats.l[row0] = sum0;
            p.stats.D[row0] = dd0;
          }
          if (in1) {
            p.stats.m[row1] = t1;
            p.stats.l[row1] = sum1;
            p.stats.D[row1] = dd1;
          }
        }
        continue;                              // no O tile to stage or store
      }
      if (leader) tma_store_wait_read();
      named_barrier(3 + g, kSoftmaxThreads);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int ch = 2 * q + h;            // 16-byte chunk (8 columns) of the row
          if (ch * 8 < p.d) {
            *reinterpret_cast<uint32_t*>(stage + r0 * kRowBytes + ((ch ^ (r0 & 7)) << 4) +
                                         j4 * 4) =
                pack_bf16x2(o[q][4 * h] * inv0, o[q][4 * h + 1] * inv0);
            *reinterpret_cast<uint32_t*>(stage + r1 * kRowBytes + ((ch ^ (r1 & 7)) << 4) +
                                         j4 * 4) =
                pack_bf16x2(o[q][4 * h + 2] * inv1, o[q][4 * h + 3] * inv1);
          }
        }
      }
      fence_proxy_async_smem();
      named_barrier(3 + g, kSoftmaxThreads);
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
inline std::atomic<int>* smem_flags_agg_bias() {
  static std::atomic<int> f[64];
  return f;
}
inline std::atomic<int>* smem_flags_bc_bias() {
  static std::atomic<int> f[64];
  return f;
}
inline std::atomic<int>* smem_flags_bc() {
  static std::atomic<int> f[64];
  return f;
}
inline std::atomic<int>* smem_flags_bc_stats() {
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
                                       float* part_u, float* part_ml, cudaStream_t st,
                                       bool pdl, const tc::BiasParams* bias = nullptr) {
  (void)a_hstride;
  using namespace tc;
  CUtensorMap mk, mv, ma;
  int a_sets = 1;
  const long long BH = (long long)B * H;
  const int box_a = n_agents > 128 ? 256 : 128;
  if (!make_map_3d(&mk, k, d, N, BH, kKeyTile) || !make_map_3d(&mv, v, d, N, BH, kKeyTile) ||
      !make_map_agents(&ma, agents, d, n_agents, H, B, a_bstride, box_a, &a_sets))
    return cudaErrorInvalidValue;
  const bool biased = bias != nullptr && bias->any();
  cudaError_t e = biased ? ensure_tc_smem(reinterpret_cast<const void*>(
                                              agent_aggregate_tc_kernel<true>),
                                          (int)kAggSmemBytes, smem_flags_agg_bias())
                         : ensure_tc_smem(reinterpret_cast<const void*>(
                                              agent_aggregate_tc_kernel<false>),
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
  p.bias = bias ? *bias : BiasParams{nullptr, 0};
  return launch_kernel(biased ? agent_aggregate_tc_kernel<true> : agent_aggregate_tc_kernel<false>,
                       dim3(plan.ctas), dim3(kThreads), kAggSmemBytes,
                       st, pdl, mk, mv, ma, a_sets, p);
}

inline cudaError_t tc_launch_broadcast(const void* q, const void* agents, long long a_bstride,
                                       const void* va, void* out, int B, int H, int N, int d,
                                       int n_agents, float c, int sm_count, cudaStream_t st,
                                       bool pdl, const tc::BiasParams* bias = nullptr,
                                       const tc::BcStats* stats = nullptr) {
  using namespace tc;
  CUtensorMap mq, ma, mva, mo;
  int a_sets = 1;
  const long long BH = (long long)B * H;
  const int kpad = round16(n_agents);
  if (!make_map_3d(&mq, q, d, N, BH, kQTile) || !make_map_3d(&mo, out, d, N, BH, kQTile) ||
      !make_map_3d(&mva, va, d, n_agents, BH, kpad) ||
      !make_map_agents(&ma, agents, d, n_agents, H, B, a_bstride, kpad, &a_sets))
    return cudaErrorInvalidValue;
  const bool biased = bias != nullptr && bias->any();
  const bool with_stats = stats != nullptr;
  if (biased && with_stats) return cudaErrorInvalidValue;   // no instantiation takes both
  const void* kernel = biased       ? reinterpret_cast<const void*>(agent_broadcast_tc_kernel<true>)
                       : with_stats ? reinterpret_cast<const void*>(
                                          agent_broadcast_tc_kernel<false, true>)
                                    : reinterpret_cast<const void*>(agent_broadcast_tc_kernel<false>);
  cudaError_t e = ensure_tc_smem(kernel, (int)kBcSmemBytes,
                                 biased       ? smem_flags_bc_bias()
                                 : with_stats ? smem_flags_bc_stats()
                                              : smem_flags_bc());
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
  p.bias = bias ? *bias : BiasParams{nullptr, 0};
  p.stats = with_stats ? *stats : BcStats{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  return launch_kernel(biased       ? agent_broadcast_tc_kernel<true>
                       : with_stats ? agent_broadcast_tc_kernel<false, true>
                                    : agent_broadcast_tc_kernel<false>,
                       dim3(p.ctas), dim3(kThreads), kBcSmemBytes, st, pdl, mq, ma, mva, mo,
                       a_sets, p);
}

}  // namespace aa
