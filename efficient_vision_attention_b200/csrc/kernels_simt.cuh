// SIMT (CUDA-core, fp32-accumulate) kernels of the Agent Attention forward pass:
//   agent_pool_kernel     adaptive average pooling of Q into agents
//   simt_attend_kernel    one online-softmax attention of a block of rows over a
//                         range of columns; serves both the aggregation
//                         (rows = agents, columns = keys, split over keys,
//                         partial output) and the broadcast (rows = queries,
//                         columns = agents, normalised output)
// These carry the fp32 path end to end (exact enough for a 1e-5 tolerance), the
// bf16 path for head dims the tensor-core kernels do not take, the agent bias
// of grids too large for the tensor-core tables, and the forward statistics of
// the backward pass.  Score blocks and P V updates are register-tiled (2 rows x
// 4 columns per thread).
#pragma once

#include "common.cuh"

namespace aa {

// ----------------------------------------------------------------- pooling
// One CTA per (slice bh, agent row py, chunk of agent columns px).  Phase 1:
// one thread per (token column x of the chunk, 8-channel group) sums that
// column over the bin's grid rows; consecutive threads read consecutive 16
// bytes, and a thread's loads (one per row, eight in flight) need a single
// trip to memory.  Phase 2: one thread per (px, channel group) adds its bin's
// column sums from shared memory and divides by the bin's token count.  Sums
// are fp32.  Writes fp32 and/or low-precision agents.
constexpr int kPoolThreads = 512;

// Agent columns per CTA, so that the chunk's token columns x channel groups
// fit in one pass of the CTA's threads (at least one agent column).
__host__ __forceinline__ int pool_px_per_cta(int grid_w, int pool_w, int d) {
  const int groups = d / 8;
  const int bin_w = (grid_w + pool_w - 1) / pool_w + 1;     // widest bin (with overlap)
  int per = kPoolThreads / (bin_w * groups);
  if (per < 1) per = 1;
  if (per > pool_w) per = pool_w;
  return per;
}

// Token columns per shared-memory window (64 KB of column sums).
__host__ __device__ __forceinline__ int pool_window_cols(int d) { return 65536 / ((d / 8) * 32); }

template <typename T>
__global__ void __launch_bounds__(kPoolThreads) agent_pool_kernel(const T* __restrict__ q,
                                                                  float* __restrict__ a_f32,
                                                                  T* __restrict__ a_lowp, int N,
                                                                  int d, int grid_h, int grid_w,
                                                                  int pool_h, int pool_w,
                                                                  int px_per_cta) {
  extern __shared__ float colsum[];          // [token column of the window][group][8]
  pdl_trigger();
  const int n_chunks = (pool_w + px_per_cta - 1) / px_per_cta;
  const int py = blockIdx.x / n_chunks;
  const int px0 = (blockIdx.x % n_chunks) * px_per_cta;
  const int px1 = min(pool_w, px0 + px_per_cta);
  const long long bh = blockIdx.y;
  const int y0 = bin_start(py, grid_h, pool_h), y1 = bin_end(py, grid_h, pool_h);
  const int xs = bin_start(px0, grid_w, pool_w), xe = bin_end(px1 - 1, grid_w, pool_w);
  const int groups = d >> 3;
  const int rows = y1 - y0;
  const T* qs = q + bh * (long long)N * d;
  const long long row_stride = (long long)grid_w * d;
  const int wcols = pool_window_cols(d);

  // phase-2 item of this thread: (px, group); there are at most kPoolThreads
  const int items2 = (px1 - px0) * groups;
  const int px = px0 + (int)threadIdx.x / groups, g2 = (int)threadIdx.x % groups;
  const bool has2 = (int)threadIdx.x < items2;
  const int bx0 = has2 ? bin_start(px, grid_w, pool_w) : 0;
  const int bx1 = has2 ? bin_end(px, grid_w, pool_w) : 0;
  float acc2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc2[i] = 0.f;

  for (int wx = xs; wx < xe; wx += wcols) {
    const int we = min(xe, wx + wcols);
    const int items = (we - wx) * groups;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
      const int x = wx + it / groups, g = it % groups;
      const T* col = qs + ((long long)y0 * grid_w + x) * d + g * 8;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      int y = 0;
      for (; y + 8 <= rows; y += 8) {      // eight independent 16-byte loads in flight
        uint4 raw[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) raw[u] = load16(col + (y + u) * row_stride);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float v[8];
          unpack8(raw[u], col + (y + u) * row_stride, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += v[i];
        }
      }
      for (; y < rows; ++y) {
        float v[8];
        load8(col + y * row_stride, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += v[i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) colsum[it * 8 + i] = acc[i];
    }
    __syncthreads();
    if (has2) {
      for (int x = max(bx0, wx); x < min(bx1, we); ++x) {
        const float* cs = colsum + ((x - wx) * groups + g2) * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc2[i] += cs[i];
      }
    }
    __syncthreads();
  }
  if (has2) {
    const long long n_agents = (long long)pool_h * pool_w;
    const float inv = 1.f / (float)((y1 - y0) * (bx1 - bx0));
    const long long off = (bh * n_agents + (long long)py * pool_w + px) * d + g2 * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float m = acc2[i] * inv;
      if (a_f32) a_f32[off + i] = m;
      if (a_lowp) a_lowp[off + i] = from_f32<T>(m);
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
  // optional agent bias added to the logits: for agent a and grid token
  // (y, x), row[h][a][y] + col[h][a][x] + block[h][a][cell(y, x)] (fp32,
  // each component may be null); cell = floor(y*pool_h/grid_h)*pool_w +
  // floor(x*pool_w/grid_w).  tok_is_col: columns are tokens (aggregation),
  // else rows are tokens (broadcast).
  const float* bias_row;
  const float* bias_col;
  const float* bias_block;
  int bias_tok_is_col;
  int grid_h, grid_w, pool_h, pool_w, n_agents;
};

__host__ __forceinline__ size_t simt_attend_smem_bytes(int d) {
  return sizeof(float) * ((size_t)kSimtRows * (d + 1) + (size_t)kSimtCols * (d + 1) +
                          (size_t)kSimtCols * d + (size_t)kSimtRows * (kSimtCols + 1) +
                          (size_t)kSimtRows * d + 3 * kSimtRows);
}

// T: element type of the column vectors, values and output; TR: element type
// of the row vectors (T, or float for fp32 rows next to bf16 columns).
template <typename T, typename TR = T>
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

  const TR* rows = static_cast<const TR*>(p.rows) +
                  agent_set_offset(bh, p.H, p.rows_bstride, p.rows_hstride);
  const T* cols = static_cast<const T*>(p.cols) +
                  agent_set_offset(bh, p.H, p.cols_bstride, p.cols_hstride);
  const T* vals = static_cast<const T*>(p.vals) +
                  agent_set_offset(bh, p.H, p.vals_bstride, p.vals_hstride);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_trigger();

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
    const bool biased = p.bias_row || p.bias_col || p.bias_block;
    // scores, register-tiled: thread t owns rows 2(t/8), +1 and columns 4(t%8) .. +3
    static_assert(kSimtRows * kSimtCols == kSimtThreads * 8, "2 x 4 scores per thread");
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int rr = 2 * (tid >> 3), jj = 4 * (tid & 7);
      const float* x0 = s_rows + rr * dp;
      const float* x1 = x0 + dp;
      const float* y0 = s_cols + jj * dp;
      for (int c = 0; c < d; ++c) {
        const float a0 = x0[c], a1 = x1[c];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float bq = y0[q * dp + c];
          sc[0][q] = fmaf(a0, bq, sc[0][q]);
          sc[1][q] = fmaf(a1, bq, sc[1][q]);
        }
      }
    }
    for (int u = 0; u < 8; ++u) {
      const int r = 2 * (tid >> 3) + (u >> 2), j = 4 * (tid & 7) + (u & 3);
      const float acc = sc[u >> 2][u & 3];
      float logit = acc * p.scale_log2;
      if (biased && r0 + r < p.n_rows && j < valid) {
        const int tok = p.bias_tok_is_col ? c0 + j : r0 + r;
        const int ag = p.bias_tok_is_col ? r0 + r : c0 + j;
        const int y = tok / p.grid_w, x = tok - y * p.grid_w;
        const long long base = (long long)(bh % p.H) * p.n_agents + ag;
        float bias = 0.f;
        if (p.bias_row) bias += p.bias_row[base * p.grid_h + y];
        if (p.bias_col) bias += p.bias_col[base * p.grid_w + x];
        if (p.bias_block) {
          const int cell = (int)(((long long)y * p.pool_h) / p.grid_h) * p.pool_w +
                           (int)(((long long)x * p.pool_w) / p.grid_w);
          bias += p.bias_block[base * ((long long)p.pool_h * p.pool_w) + cell];
        }
        logit = fmaf(bias, kLog2e, logit);
      }
      s_p[r * (kSimtCols + 1) + j] = logit;
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
    // U = alpha U + P V, register-tiled: items (row pair, 4 channels)
    {
      const int nq = (d + 3) >> 2;
      for (int e = tid; e < (kSimtRows / 2) * nq; e += kSimtThreads) {
        const int rp = e / nq, c = 4 * (e - rp * nq);
        const int r = 2 * rp;
        const float* p0 = s_p + r * (kSimtCols + 1);
        const float* p1 = p0 + (kSimtCols + 1);
        float a0[4], a1[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          a0[q] = (c + q < d) ? s_u[r * d + c + q] * s_alpha[r] : 0.f;
          a1[q] = (c + q < d) ? s_u[(r + 1) * d + c + q] * s_alpha[r + 1] : 0.f;
        }
        for (int j = 0; j < valid; ++j) {
          const float w0 = p0[j], w1 = p1[j];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float m = (c + q < d) ? s_vals[j * d + c + q] : 0.f;
            a0[q] = fmaf(w0, m, a0[q]);
            a1[q] = fmaf(w1, m, a1[q]);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (c + q < d) {
            s_u[r * d + c + q] = a0[q];
            s_u[(r + 1) * d + c + q] = a1[q];
          }
        }
      }
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

}  // namespace aa
