// Backward pass of the Agent Attention forward pass (SIMT, fp32 arithmetic),
// for finetuning through both softmax stages.  With
//   P1 = softmax_rows(s A K^T) (k x N), V_A = P1 V,
//   P2 = softmax_rows(s Q A^T) (N x k), O = P2 V_A
// and an output gradient dO:
//   bwd_query_kernel  per query row i: P2_i (two passes over agent chunks for
//                     its max and sum, or one when the tensor-core broadcast
//                     supplied them with D_i and the bf16 exponentials, which
//                     then replace the score dot products), dP2_ij = dO_i .
//                     V_A_j, D_i = sum_j P2_ij dP2_ij, dS2 = P2 (dP2 - D_i);
//                     writes dQ_i = s sum_j dS2_ij A_j (fp32) and adds the
//                     CTA's sums of
//                     P2_ij dO_i (-> dV_A_j) and s dS2_ij Q_i (-> dA_j) into
//                     global fp32 accumulators.
//   bwd_key_kernel    per key row n: P1_jn from the aggregation's stored row
//                     max and sum (the exponentials from a tensor-core pass
//                     over K when given), dP1_jn = dV_A_j . V_n, dS1 = P1
//                     (dP1 - E_j)
//                     with E_j = dV_A_j . V_A_j; writes dK_n = s sum_j dS1_jn
//                     A_j and dV_n = sum_j P1_jn dV_A_j and adds s dS1_jn K_n
//                     into dA_j.
//   bwd_finish_kernel dQ += the pooling adjoint of dA (each token gets dA of
//                     every bin holding it divided by the bin's size), in the
//                     output dtype.
// Scores are in log2 units (scale * log2 e), like the forward kernels.
#pragma once

#include "common.cuh"

namespace aa {

constexpr int kBwdRows = 64;     // query or key rows per CTA
constexpr int kBwdCols = 32;     // agents per chunk
constexpr int kBwdThreads = 256;
// Row stride of the [rows][agents] score and gradient tiles: 36 floats, so a
// row's 4 consecutive agents are one aligned float4 and the 4 row pairs a
// warp writes in bwd_dots fall in 4 disjoint groups of 8 banks.
constexpr int kBwdTStride = kBwdCols + 4;

struct BwdArgs {
  const void* x;        // q (query kernel) or k (key kernel): [BH][N][d] of T
  const void* y;        // dO (query kernel) or v (key kernel): [BH][N][d] of T
  const float* a;       // agents [BH][n_agents][d] fp32
  const float* va;      // V_A [BH][n_agents][d] fp32
  const float* dva;     // key kernel: dV_A [BH][n_agents][d]
  const float* ml;      // key kernel: aggregation row max (log2 units) and sum [BH][n_agents][2]
  const float* e;       // key kernel: E_j = dV_A_j . V_A_j [BH][n_agents]
  const float* st_m;    // query kernel, or null: each query's score max (log2 units),
  const float* st_l;    //   sum of 2^(s - m) and D = dO . O [BH][N], computed
  const float* st_D;    //   beforehand (then the first sweep is skipped)
  const uint32_t* st_p; // or null: 2^(s - m) as bf16 pairs, [BH][N][st_kpad] bf16 (even;
  int st_kpad;          //   columns >= n_agents hold 0): the query kernel's with st_m (m
                        //   the query's max), the key kernel's with m the agent's max
  float* dq;            // query kernel: dQ [BH][N][d] fp32
  float* dva_acc;       // query kernel: += dV_A
  float* da_acc;        // both: += dA
  void* dk;             // key kernel: dK [BH][N][d] of T
  void* dv;             // key kernel: dV [BH][N][d] of T
  int N, n_agents, d;
  float scale;          // s
  float scale_log2;     // s * log2 e
};

// Row stride of the staged [rows][d] tiles: d + 4 floats, so every row starts
// on a 16-byte boundary (float4 reads along the channels) and consecutive
// rows start 4 banks apart.
__host__ __device__ __forceinline__ int bwd_row_stride(int d) { return d + 4; }

// Shared memory of bwd_query_kernel<T, true> (dQ accumulated in registers,
// d <= 64): the staged tiles and the row statistics only.
__host__ __forceinline__ size_t bwd_query_reg_smem_bytes(int d) {
  const size_t dp = bwd_row_stride(d);
  return sizeof(float) * (2 * kBwdRows * dp + 2 * kBwdCols * dp + 2 * kBwdRows * kBwdTStride +
                          4 * kBwdRows);
}
__host__ __forceinline__ size_t bwd_smem_bytes(int d) {
  const size_t dp = bwd_row_stride(d);
  return sizeof(float) * (2 * kBwdRows * dp + 2 * kBwdCols * dp + 2 * kBwdRows * kBwdTStride +
                          (size_t)kBwdRows * dp * 2 + 4 * kBwdRows + 4 * kBwdCols);
}

template <typename T>
__device__ __forceinline__ void bwd_load_rows(float* dst, const T* src, int r0, int n_rows, int d,
                                              int dp) {
  for (int e = threadIdx.x; e < kBwdRows * d; e += kBwdThreads) {
    const int r = e / d, c = e - r * d;
    dst[r * dp + c] = (r0 + r < n_rows) ? to_f32(src[(long long)(r0 + r) * d + c]) : 0.f;
  }
}

__device__ __forceinline__ void bwd_load_agents(float* dst, const float* src, int j0, int n_agents,
                                                int d, int dp) {
  for (int e = threadIdx.x; e < kBwdCols * d; e += kBwdThreads) {
    const int j = e / d, c = e - j * d;
    dst[j * dp + c] = (j0 + j < n_agents) ? src[(long long)(j0 + j) * d + c] : 0.f;
  }
}

// dot products of the CTA's rows with a chunk's agents: out[r][j] = X_r . Y_j * mul.
// Register-tiled on the first 128 threads: thread t owns rows t/8 + 16i and
// agents t%8 + 8q, i, q = 0..3 (128 threads x 16 dots = 64 x 32); per 4
// channels it reads 8 float4 (rows 16-byte aligned, d % 4 == 0) for 64 FMAs.
// The 8 threads of a quarter-warp read 8 consecutive agent rows d + 4 floats
// apart: 8 distinct 4-bank groups (no conflict), and a warp's 4 row groups
// read 4 consecutive rows (also distinct bank groups; rows 4 apart would
// collide in pairs for d + 4 = 44); the threads sharing a row get a
// broadcast.  (Shared-memory reads bound these kernels: 8 reads per 64 FMAs
// instead of 6 per 32 with all 256 threads on 2 x 4 tiles.)
__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}
__device__ __forceinline__ void bwd_dots(float* out, const float* X, const float* Y, int d, int dp,
                                         float mul) {
  static_assert(kBwdRows == 64 && kBwdCols == 32, "4 x 4 dots per thread on 128 threads");
  const int t = threadIdx.x;
  if (t >= 128) return;
  const int r = t >> 3, j = t & 7;
  const float* x0 = X + r * dp;
  const float* y0 = Y + j * dp;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
  for (int c = 0; c < d; c += 4) {
    float4 a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(x0 + 16 * i * dp + c);
#pragma unroll
    for (int q = 0; q < 4; ++q) b[q] = *reinterpret_cast<const float4*>(y0 + 8 * q * dp + c);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = dot4(a[i], b[q], acc[i][q]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) out[(r + 16 * i) * kBwdTStride + j + 8 * q] = acc[i][q] * mul;
}

// out[r][c] += mul * sum_{j < valid} W[r][j] M[j][c] for the CTA's 64 rows:
// thread items = (row pair, 4 channels); per 4 agents, one float4 of W per
// row and one float4 of M per agent feed 32 FMAs (6 shared reads).  Agents
// past `valid` up to the next multiple of 4 have zero W (and zero M rows).
__device__ __forceinline__ void bwd_rows_acc(float* out, const float* W, const float* M, int d,
                                             int dp, int valid, float mul) {
  const int nq = (d + 3) >> 2;
  for (int e = threadIdx.x; e < (kBwdRows / 2) * nq; e += kBwdThreads) {
    const int rp = e / nq, c = 4 * (e - rp * nq);
    const int r = 2 * rp;
    float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < valid; j += 4) {
      const float4 w0 = *reinterpret_cast<const float4*>(W + r * kBwdTStride + j);
      const float4 w1 = *reinterpret_cast<const float4*>(W + (r + 1) * kBwdTStride + j);
      const float wa[4] = {w0.x, w0.y, w0.z, w0.w}, wb[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 m4 = *reinterpret_cast<const float4*>(M + (j + q) * dp + c);   // d % 4 == 0
        const float m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a0[i] = fmaf(wa[q], m[i], a0[i]);
          a1[i] = fmaf(wb[q], m[i], a1[i]);
        }
      }
    }
    // out rows dp floats apart (16-byte aligned): one float4 update per row
    float4* o0 = reinterpret_cast<float4*>(out + r * dp + c);
    float4* o1 = reinterpret_cast<float4*>(out + (r + 1) * dp + c);
    float4 u0 = *o0, u1 = *o1;
    u0.x += mul * a0[0]; u0.y += mul * a0[1]; u0.z += mul * a0[2]; u0.w += mul * a0[3];
    u1.x += mul * a1[0]; u1.y += mul * a1[1]; u1.z += mul * a1[2]; u1.w += mul * a1[3];
    *o0 = u0;
    *o1 = u1;
  }
}

// acc[i][e] += sum_{j < valid} W[rq + 16 i][j] M[j][c + e] for the CTA's 64
// rows held in registers across the agent chunks (d <= 64): thread t < 16 nq
// owns rows rq + 16 i (i = 0..3, rq = t / nq) and channels c = 4 (t % nq) ..
// + 3; per 4 agents, 4 float4 of W and 4 of M feed 64 FMAs.  Agents past
// `valid` up to the next multiple of 4 have zero W (and zero M rows).  A
// warp's row groups read consecutive rows (distinct bank groups).
__device__ __forceinline__ void bwd_rows_acc_reg(float (&acc)[4][4], const float* W,
                                                 const float* M, int d, int dp, int valid) {
  const int nq = d >> 2;
  const int t = threadIdx.x;
  if (t >= 16 * nq) return;
  const int rq = t / nq, c = 4 * (t - rq * nq);
  for (int j = 0; j < valid; j += 4) {
    float4 w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = *reinterpret_cast<const float4*>(W + (rq + 16 * i) * kBwdTStride + j);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 m4 = *reinterpret_cast<const float4*>(M + (j + q) * dp + c);
      const float m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float wq = q == 0 ? w[i].x : q == 1 ? w[i].y : q == 2 ? w[i].z : w[i].w;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = fmaf(wq, m[e], acc[i][e]);
      }
    }
  }
}

// out[r][c] += mul * sum_{j < valid} W[r][j] M[j][c] for d <= 64 on 4 x 4
// register tiles (rows rq + 16 i, channels c..c+3: 8 shared reads per 64
// FMAs, against 6 per 32 in bwd_rows_acc), added into the shared rows once
// per chunk.
__device__ __forceinline__ void bwd_rows_acc_tile(float* out, const float* W, const float* M,
                                                  int d, int dp, int valid, float mul) {
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  bwd_rows_acc_reg(acc, W, M, d, dp, valid);
  const int nq = d >> 2;
  const int t = threadIdx.x;
  if (t >= 16 * nq) return;
  const int rq = t / nq, c = 4 * (t - rq * nq);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4* o = reinterpret_cast<float4*>(out + (rq + 16 * i) * dp + c);
    float4 u = *o;
    u.x += mul * acc[i][0];
    u.y += mul * acc[i][1];
    u.z += mul * acc[i][2];
    u.w += mul * acc[i][3];
    *o = u;
  }
}

// Four consecutive floats added into global memory by one vector reduction
// (16-byte aligned address): a quarter of the L2 atomic operations of four
// scalar atomicAdds.
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float e) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(e)
               : "memory");
}

// acc[j][c] = mul * sum_r W[r][j] X[r][c] for the chunk's agents j < valid,
// added atomically into dst[(j0 + j) * d + c].  Items = (4 agents, 4
// channels): per row one float4 of W (the 4 agents) and one of X (the 4
// channels) feed 16 FMAs.  The 64 rows are split between up to 3 groups of
// items (as many as the block holds), each adding its own partial sums.
constexpr int kBwdAccGroups = 3;
__device__ __forceinline__ void bwd_agents_acc(float* dst, int j0, const float* W, const float* X,
                                               int d, int dp, int valid, float mul) {
  const int nq = d >> 2;                       // d % 8 == 0
  const int items = (kBwdCols / 4) * nq;
  const int groups = min(kBwdAccGroups, kBwdThreads / items);
  const int t = threadIdx.x;
  if (t >= groups * items) return;
  const int grp = t / items, it = t - grp * items;
  const int jq = it / nq, c = 4 * (it - jq * nq);
  const int j = 4 * jq;
  if (j >= valid) return;
  const int rb = grp * kBwdRows / groups, re = (grp + 1) * kBwdRows / groups;
  float a[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int e = 0; e < 4; ++e) a[q][e] = 0.f;
  for (int r = rb; r < re; ++r) {
    const float4 w4 = *reinterpret_cast<const float4*>(W + r * kBwdTStride + j);
    const float4 x4 = *reinterpret_cast<const float4*>(X + r * dp + c);
    const float w[4] = {w4.x, w4.y, w4.z, w4.w}, x[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) a[q][e] = fmaf(w[q], x[e], a[q][e]);
  }
  // W is zero for agents >= valid (the chunk's tail), but their rows of dst
  // may not exist
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (j + q < valid)
      red_add_v4(dst + (long long)(j0 + j + q) * d + c, mul * a[q][0], mul * a[q][1],
                 mul * a[q][2], mul * a[q][3]);
}

// kRegAcc (d <= 64): the dQ accumulator lives in registers (no shared
// accumulator; 80 registers, 3 CTAs per SM: bounding it to 4 CTAs at 64
// registers spilled and measured slower).
template <typename T, bool kRegAcc = false>
__global__ void __launch_bounds__(kBwdThreads, kRegAcc ? 3 : 1) bwd_query_kernel(BwdArgs p) {
  extern __shared__ float sm[];
  const int d = p.d, dp = bwd_row_stride(d);
  float* s_x = sm;                                   // Q rows [64][d+4]
  float* s_y = s_x + kBwdRows * dp;                  // dO rows
  float* s_a = s_y + kBwdRows * dp;                  // agent chunk [32][d+4]
  float* s_va = s_a + kBwdCols * dp;
  float* s_t = s_va + kBwdCols * dp;                 // scores / P2 [64][36]
  float* s_g = s_t + kBwdRows * kBwdTStride;      // dP2 / dS2 [64][36]
  float* s_acc = s_g + kBwdRows * kBwdTStride;    // dQ accumulator [64][d+4] (not kRegAcc)
  float* s_m = kRegAcc ? s_acc : s_acc + kBwdRows * dp;
  float racc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) racc[i][e] = 0.f;
  float* s_l = s_m + kBwdRows;
  float* s_D = s_l + kBwdRows;
  const long long bh = blockIdx.y;
  const int r0 = blockIdx.x * kBwdRows;
  const int n_rows = p.N, K = p.n_agents;
  const T* X = static_cast<const T*>(p.x) + bh * (long long)p.N * d;
  const T* Y = static_cast<const T*>(p.y) + bh * (long long)p.N * d;
  const float* A = p.a + bh * (long long)K * d;
  const float* VA = p.va + bh * (long long)K * d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bwd_load_rows(s_x, X, r0, n_rows, d, dp);
  bwd_load_rows(s_y, Y, r0, n_rows, d, dp);
  if (!kRegAcc)
    for (int e = tid; e < kBwdRows * dp; e += kBwdThreads) s_acc[e] = 0.f;
  const bool given = p.st_m != nullptr;
  for (int r = tid; r < kBwdRows; r += kBwdThreads) {
    const bool in = r0 + r < n_rows;
    const long long i = bh * (long long)n_rows + r0 + r;
    s_m[r] = given ? (in ? p.st_m[i] : 0.f) : -INFINITY;
    s_l[r] = given ? (in ? p.st_l[i] : 1.f) : 0.f;
    s_D[r] = given ? (in ? p.st_D[i] : 0.f) : 0.f;
  }
  __syncthreads();
  // pass 1 (online over the chunks, unless the statistics are given): each
  // row's score max m and sum l = sum_j 2^(s_j - m), and D~ = sum_j 2^(s_j -
  // m) (dO . V_A_j), both rescaled when m grows; D_i = D~ / l
  for (int j0 = 0; j0 < (given ? 0 : K); j0 += kBwdCols) {
    const int valid = min(kBwdCols, K - j0);
    bwd_load_agents(s_a, A, j0, K, d, dp);
    bwd_load_agents(s_va, VA, j0, K, d, dp);
    __syncthreads();
    bwd_dots(s_t, s_x, s_a, d, dp, p.scale_log2);
    bwd_dots(s_g, s_y, s_va, d, dp, 1.f);
    __syncthreads();
    for (int r = warp; r < kBwdRows; r += kBwdThreads / 32) {
      const float t = lane < valid ? s_t[r * kBwdTStride + lane] : -INFINITY;
      float mx = t;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(s_m[r], mx);
      float e = lane < valid ? exp2f(t - m_new) : 0.f;
      float eg = lane < valid ? e * s_g[r * kBwdTStride + lane] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        e += __shfl_xor_sync(0xffffffffu, e, o);
        eg += __shfl_xor_sync(0xffffffffu, eg, o);
      }
      if (lane == 0) {
        const float rs = exp2f(s_m[r] - m_new);   // 0 on the first chunk (s_m = -inf)
        s_l[r] = s_l[r] * rs + e;
        s_D[r] = s_D[r] * rs + eg;
        s_m[r] = m_new;
      }
    }
    __syncthreads();
  }
  if (!given) {
    for (int r = tid; r < kBwdRows; r += kBwdThreads) s_D[r] = s_D[r] / s_l[r];
    __syncthreads();
  }
  // pass 2: dS2, dQ, and the chunk's contributions to dV_A and dA.  With
  // the exponentials given, P2 = 2^(s - m) / l comes from them (thread items
  // = 4 bf16 pairs: rows e / 16, agents 2 (e % 16), e = tid + 256 i) and the
  // score dot products are skipped.
  float* dva = p.dva_acc + bh * (long long)K * d;
  float* da = p.da_acc + bh * (long long)K * d;
  static_assert(kBwdRows * kBwdCols == 8 * kBwdThreads, "4 P pairs per thread");
  const bool p_given = p.st_p != nullptr;
  const uint32_t* Pw = p_given ? p.st_p + (bh * n_rows + r0) * (long long)(p.st_kpad / 2) : nullptr;
  for (int j0 = 0; j0 < K; j0 += kBwdCols) {
    const int valid = min(kBwdCols, K - j0);
    uint32_t pw[4] = {0u, 0u, 0u, 0u};
    if (p_given) {                     // issued before the dot products hide the latency
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = tid + kBwdThreads * i, r = e >> 4, j = 2 * (e & 15);
        if (j < valid && r0 + r < n_rows)
          pw[i] = __ldg(Pw + (long long)r * (p.st_kpad / 2) + ((j0 + j) >> 1));
      }
    }
    bwd_load_agents(s_a, A, j0, K, d, dp);
    bwd_load_agents(s_va, VA, j0, K, d, dp);
    __syncthreads();
    if (!p_given) bwd_dots(s_t, s_x, s_a, d, dp, p.scale_log2);
    bwd_dots(s_g, s_y, s_va, d, dp, 1.f);
    __syncthreads();
    if (p_given) {
      // a pair's second agent past the chunk is a padding column (0)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = tid + kBwdThreads * i, r = e >> 4, j = 2 * (e & 15);
        const float inv = 1.f / s_l[r], Dr = s_D[r];
        const float2 g2 = *reinterpret_cast<const float2*>(s_g + r * kBwdTStride + j);
        const float p0 = __uint_as_float(pw[i] << 16) * inv;           // bf16 -> fp32
        const float p1 = __uint_as_float(pw[i] & 0xffff0000u) * inv;
        *reinterpret_cast<float2*>(s_t + r * kBwdTStride + j) = make_float2(p0, p1);
        *reinterpret_cast<float2*>(s_g + r * kBwdTStride + j) =
            make_float2(p0 * (g2.x - Dr), p1 * (g2.y - Dr));
      }
    } else {
      for (int e = tid; e < kBwdRows * kBwdCols; e += kBwdThreads) {
        const int r = e / kBwdCols, j = e - r * kBwdCols;
        float pr = 0.f, ds = 0.f;
        if (j < valid && r0 + r < n_rows) {
          pr = exp2f(s_t[r * kBwdTStride + j] - s_m[r]) / s_l[r];
          ds = pr * (s_g[r * kBwdTStride + j] - s_D[r]);
        }
        s_t[r * kBwdTStride + j] = pr;
        s_g[r * kBwdTStride + j] = ds;
      }
    }
    __syncthreads();
    if constexpr (kRegAcc)                                      // dQ_r += sum_j ds A_j
      bwd_rows_acc_reg(racc, s_g, s_a, d, dp, valid);
    else
      bwd_rows_acc(s_acc, s_g, s_a, d, dp, valid, p.scale);     // dQ_r += s sum_j ds A_j
    bwd_agents_acc(dva, j0, s_t, s_y, d, dp, valid, 1.f);       // dV_A_j += sum_r P2 dO_r
    bwd_agents_acc(da, j0, s_g, s_x, d, dp, valid, p.scale);    // dA_j += s sum_r dS2 Q_r
    __syncthreads();
  }
  float* dq = p.dq + bh * (long long)p.N * d;
  if constexpr (kRegAcc) {
    const int nq = d >> 2;
    if (tid < 16 * nq) {
      const int rq = tid / nq, c = 4 * (tid - rq * nq);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rq + 16 * i;
        if (r0 + r < n_rows)
          *reinterpret_cast<float4*>(dq + (long long)(r0 + r) * d + c) =
              make_float4(p.scale * racc[i][0], p.scale * racc[i][1], p.scale * racc[i][2],
                          p.scale * racc[i][3]);
      }
    }
  } else {
    for (int e = tid; e < kBwdRows * d; e += kBwdThreads) {
      const int r = e / d, c = e - r * d;
      if (r0 + r < n_rows) dq[(long long)(r0 + r) * d + c] = s_acc[r * dp + c];
    }
  }
}

// Three CTAs per SM (the shared-memory limit too): the given-exponential path
// would otherwise take 110 registers and two.
template <typename T>
__global__ void __launch_bounds__(kBwdThreads, 3) bwd_key_kernel(BwdArgs p) {
  extern __shared__ float sm[];
  const int d = p.d, dp = bwd_row_stride(d);
  float* s_x = sm;                                   // K rows
  float* s_y = s_x + kBwdRows * dp;                  // V rows
  float* s_a = s_y + kBwdRows * dp;                  // agent chunk
  float* s_dva = s_a + kBwdCols * dp;                // dV_A chunk
  float* s_t = s_dva + kBwdCols * dp;                // P1 [64][36]
  float* s_g = s_t + kBwdRows * kBwdTStride;      // dS1 [64][36]
  float* s_dk = s_g + kBwdRows * kBwdTStride;     // [64][d+4]
  float* s_dv = s_dk + kBwdRows * dp;                // [64][d+4]
  float* s_jm = s_dv + kBwdRows * dp;                // chunk: row max, sum, E (3 x 32)
  float* s_jl = s_jm + kBwdCols;
  float* s_je = s_jl + kBwdCols;
  const long long bh = blockIdx.y;
  const int r0 = blockIdx.x * kBwdRows;
  const int n_rows = p.N, K = p.n_agents;
  const T* X = static_cast<const T*>(p.x) + bh * (long long)p.N * d;
  const T* Y = static_cast<const T*>(p.y) + bh * (long long)p.N * d;
  const float* A = p.a + bh * (long long)K * d;
  const float* DVA = p.dva + bh * (long long)K * d;
  const float* ML = p.ml + bh * (long long)K * 2;
  const float* EJ = p.e + bh * (long long)K;
  float* da = p.da_acc + bh * (long long)K * d;
  const int tid = threadIdx.x;
  bwd_load_rows(s_x, X, r0, n_rows, d, dp);
  bwd_load_rows(s_y, Y, r0, n_rows, d, dp);
  for (int e = tid; e < kBwdRows * dp; e += kBwdThreads) {
    s_dk[e] = 0.f;
    s_dv[e] = 0.f;
  }
  // With the exponentials given (the broadcast run over K, each agent's max
  // subtracted), P1 = 2^(s - m_j) / l_j comes from them (thread items = 4
  // bf16 pairs: rows e / 16, agents 2 (e % 16), e = tid + 256 i) and the
  // score dot products are skipped.
  const bool p_given = p.st_p != nullptr;
  const uint32_t* Pw = p_given ? p.st_p + (bh * n_rows + r0) * (long long)(p.st_kpad / 2) : nullptr;
  for (int j0 = 0; j0 < K; j0 += kBwdCols) {
    const int valid = min(kBwdCols, K - j0);
    uint32_t pw[4] = {0u, 0u, 0u, 0u};
    if (p_given) {                     // issued before the dot products hide the latency
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = tid + kBwdThreads * i, r = e >> 4, j = 2 * (e & 15);
        if (j < valid && r0 + r < n_rows)
          pw[i] = __ldg(Pw + (long long)r * (p.st_kpad / 2) + ((j0 + j) >> 1));
      }
    }
    __syncthreads();
    bwd_load_agents(s_a, A, j0, K, d, dp);
    bwd_load_agents(s_dva, DVA, j0, K, d, dp);
    // the chunk's E_j (computed once per slice by bwd_agent_e_kernel) and
    // the saved aggregation statistics
    for (int j = tid; j < kBwdCols; j += kBwdThreads) {
      s_je[j] = j < valid ? EJ[j0 + j] : 0.f;
      s_jm[j] = j < valid ? ML[(long long)(j0 + j) * 2] : 0.f;
      s_jl[j] = j < valid ? ML[(long long)(j0 + j) * 2 + 1] : 1.f;
    }
    __syncthreads();
    if (!p_given) bwd_dots(s_t, s_x, s_a, d, dp, p.scale_log2);
    bwd_dots(s_g, s_y, s_dva, d, dp, 1.f);
    __syncthreads();
    if (p_given) {
      // padding agents (j >= valid) have l = 1, E = 0 and zero words
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = tid + kBwdThreads * i, r = e >> 4, j = 2 * (e & 15);
        const float2 g2 = *reinterpret_cast<const float2*>(s_g + r * kBwdTStride + j);
        const float p0 = __uint_as_float(pw[i] << 16) / s_jl[j];             // bf16 -> fp32
        const float p1 = __uint_as_float(pw[i] & 0xffff0000u) / s_jl[j + 1];
        *reinterpret_cast<float2*>(s_t + r * kBwdTStride + j) = make_float2(p0, p1);
        *reinterpret_cast<float2*>(s_g + r * kBwdTStride + j) =
            make_float2(p0 * (g2.x - s_je[j]), p1 * (g2.y - s_je[j + 1]));
      }
    } else {
      for (int e = tid; e < kBwdRows * kBwdCols; e += kBwdThreads) {
        const int r = e / kBwdCols, j = e - r * kBwdCols;
        float pr = 0.f, ds = 0.f;
        if (j < valid && r0 + r < n_rows) {
          pr = exp2f(s_t[r * kBwdTStride + j] - s_jm[j]) / s_jl[j];
          ds = pr * (s_g[r * kBwdTStride + j] - s_je[j]);
        }
        s_t[r * kBwdTStride + j] = pr;
        s_g[r * kBwdTStride + j] = ds;
      }
    }
    __syncthreads();
    if (d <= 64) {                                              // 16 (d / 4) <= 256 threads
      bwd_rows_acc_tile(s_dk, s_g, s_a, d, dp, valid, p.scale);   // dK_r += s sum_j dS1 A_j
      bwd_rows_acc_tile(s_dv, s_t, s_dva, d, dp, valid, 1.f);     // dV_r += sum_j P1 dV_A_j
    } else {
      bwd_rows_acc(s_dk, s_g, s_a, d, dp, valid, p.scale);
      bwd_rows_acc(s_dv, s_t, s_dva, d, dp, valid, 1.f);
    }
    bwd_agents_acc(da, j0, s_g, s_x, d, dp, valid, p.scale);    // dA_j += s sum_r dS1 K_r
  }
  __syncthreads();
  T* dk = static_cast<T*>(p.dk) + bh * (long long)p.N * d;
  T* dv = static_cast<T*>(p.dv) + bh * (long long)p.N * d;
  for (int e = tid; e < kBwdRows * d; e += kBwdThreads) {
    const int r = e / d, c = e - r * d;
    if (r0 + r < n_rows) {
      dk[(long long)(r0 + r) * d + c] = from_f32<T>(s_dk[r * dp + c]);
      dv[(long long)(r0 + r) * d + c] = from_f32<T>(s_dv[r * dp + c]);
    }
  }
}

// E_j = dV_A_j . V_A_j for every (slice, agent): a warp per agent row.
__global__ void __launch_bounds__(256) bwd_agent_e_kernel(const float* __restrict__ dva,
                                                          const float* __restrict__ va,
                                                          float* __restrict__ e, long long rows,
                                                          int d) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < d; c += 32) acc = fmaf(dva[row * d + c], va[row * d + c], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) e[row] = acc;
}

// dQ = dq_acc (+ the pooling adjoint of dA when the agents were pooled), in T.
// Thread per (token, 8-channel group); grid (ceil(N*d/8 / 256), BH).  The
// bins holding a token are found once per axis: the floor cell c = y P / G
// and its two neighbours are the only candidates (adaptive bins overlap by at
// most one token), and a token lies in one or two bins per axis.  Each bin
// adds its dA row divided by the bin's token count.
template <typename T>
__global__ void __launch_bounds__(256) bwd_finish_kernel(const float* __restrict__ dq_acc,
                                                         const float* __restrict__ da, T* dq,
                                                         int N, int d, int grid_h, int grid_w,
                                                         int pool_h, int pool_w, int pooled) {
  // the adaptive bins' bounds along each axis, once per block (pool sides
  // <= 256: k <= 256)
  __shared__ int s_by[2][256], s_bx[2][256];
  if (pooled) {
    for (int i = threadIdx.x; i < pool_h; i += blockDim.x) {
      s_by[0][i] = bin_start(i, grid_h, pool_h);
      s_by[1][i] = bin_end(i, grid_h, pool_h);
    }
    for (int i = threadIdx.x; i < pool_w; i += blockDim.x) {
      s_bx[0][i] = bin_start(i, grid_w, pool_w);
      s_bx[1][i] = bin_end(i, grid_w, pool_w);
    }
    __syncthreads();
  }
  const long long bh = blockIdx.y;
  const int groups = d >> 3;
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)N * groups) return;
  // 32-bit divisions when the index products fit (every grid below 46341
  // tokens a side)
  const bool f32 = (long long)N * groups <= 0x7fffffffLL &&
                   (long long)grid_h * pool_h <= 0x7fffffffLL &&
                   (long long)grid_w * pool_w <= 0x7fffffffLL;
  const int n = f32 ? (int)e / groups : (int)(e / groups);
  const int g = (int)(e - (long long)n * groups);
  const long long off = (bh * N + n) * (long long)d + g * 8;
  const float4 s0 = *reinterpret_cast<const float4*>(dq_acc + off);
  const float4 s1 = *reinterpret_cast<const float4*>(dq_acc + off + 4);
  float acc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  if (pooled) {
    const int y = n / grid_w, x = n - y * grid_w;
    // first and last bin holding the token along each axis, with their sizes
    int by0 = -1, by1 = -1, sy0 = 1, sy1 = 1, bx0 = -1, bx1 = -1, sx0 = 1, sx1 = 1;
    const int cy = f32 ? (y * pool_h) / grid_h : (int)(((long long)y * pool_h) / grid_h);
    const int cx = f32 ? (x * pool_w) / grid_w : (int)(((long long)x * pool_w) / grid_w);
    for (int py = max(0, cy - 1); py <= min(pool_h - 1, cy + 1); ++py) {
      const int y0 = s_by[0][py], y1 = s_by[1][py];
      if (y >= y0 && y < y1) {
        if (by0 < 0) {
          by0 = py;
          sy0 = y1 - y0;
        } else {
          by1 = py;
          sy1 = y1 - y0;
        }
      }
    }
    for (int px = max(0, cx - 1); px <= min(pool_w - 1, cx + 1); ++px) {
      const int x0 = s_bx[0][px], x1 = s_bx[1][px];
      if (x >= x0 && x < x1) {
        if (bx0 < 0) {
          bx0 = px;
          sx0 = x1 - x0;
        } else {
          bx1 = px;
          sx1 = x1 - x0;
        }
      }
    }
    const float* D = da + bh * (long long)pool_h * pool_w * d + g * 8;
#pragma unroll
    for (int iy = 0; iy < 2; ++iy) {
      const int py = iy ? by1 : by0, hy = iy ? sy1 : sy0;
#pragma unroll
      for (int ix = 0; ix < 2; ++ix) {
        const int px = ix ? bx1 : bx0, hx = ix ? sx1 : sx0;
        if (py < 0 || px < 0) continue;
        const float* row = D + ((long long)py * pool_w + px) * d;
        const float4 d0 = *reinterpret_cast<const float4*>(row);
        const float4 d1 = *reinterpret_cast<const float4*>(row + 4);
        const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
        const float size = (float)(hy * hx);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += dv[i] / size;
      }
    }
  }
  T* o = dq + off;                           // 16-byte aligned: d % 8 == 0
  if constexpr (sizeof(T) == 4) {
    reinterpret_cast<float4*>(o)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(o)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  } else {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(o) = *reinterpret_cast<const uint4*>(h);
  }
}

}  // namespace aa
