// Host side of the Agent Attention C ABI (include/agent_attn.h): argument
// validation, scratch layout, kernel selection and launch sequencing.
//
// Launch sequence of one forward pass on `stream`:
//   agent_pool (skipped for learnable agents)
//   -> agent_aggregate (split over keys; partial U, running max, running sum)
//   -> agent_merge (log-sum-exp merge of the splits into V_A)
//   -> agent_broadcast
// bf16 problems with d <= 64 run the tcgen05/TMA tensor-core kernels for the
// aggregation and the broadcast; every other problem runs the SIMT kernels.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "agent_attn.h"
#include "common.cuh"
#include "kernels_bwd.cuh"
#include "kernels_dwc.cuh"
#include "kernels_merge.cuh"
#include "kernels_pool.cuh"
#include "kernels_simt.cuh"
#include "kernels_tc.cuh"
#include "kernels_fused.cuh"

namespace aa {
namespace {

thread_local char g_cuda_err[384] = "AA_ERR_CUDA: no CUDA error recorded on this thread";

int cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_cuda_err, sizeof(g_cuda_err), "AA_ERR_CUDA: %s: %s (%s)", what, cudaGetErrorName(e),
           cudaGetErrorString(e));
  // a launch error is also left as the thread's last error; clear it (it is
  // reported here) so that the next call's launch checks do not see it again
  (void)cudaGetLastError();
  return AA_ERR_CUDA;
}
#define AA_CUDA(call)                                   \
  do {                                                  \
    cudaError_t _e = (call);                            \
    if (_e != cudaSuccess) return cuda_fail(_e, #call); \
  } while (0)

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

int device_sm_count(int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= 0 && dev < kMaxDevices) {
    int c = g_sm_count[dev].load(std::memory_order_relaxed);
    if (c > 0) {
      *out = c;
      return AA_OK;
    }
  }
  int c = 0;
  e = cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
  if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(c, std::memory_order_relaxed);
  *out = c;
  return AA_OK;
}

// Library-owned stream-ordered memory pool per device.  Freed scratch stays
// in the pool (release threshold = max) so that repeated calls do not map and
// unmap device memory; the pool is created on first use on each device.
std::atomic<cudaMemPool_t> g_pool[kMaxDevices];

int device_pool(cudaMemPool_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    e = cudaDeviceGetDefaultMemPool(out, dev);
    return e == cudaSuccess ? AA_OK : cuda_fail(e, "cudaDeviceGetDefaultMemPool");
  }
  cudaMemPool_t p = g_pool[dev].load(std::memory_order_acquire);
  if (p != nullptr) {
    *out = p;
    return AA_OK;
  }
  cudaMemPoolProps props;
  memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.handleTypes = cudaMemHandleTypeNone;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t fresh = nullptr;
  e = cudaMemPoolCreate(&fresh, &props);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
  unsigned long long keep = ~0ull;
  e = cudaMemPoolSetAttribute(fresh, cudaMemPoolAttrReleaseThreshold, &keep);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolSetAttribute");
  cudaMemPool_t expected = nullptr;
  if (!g_pool[dev].compare_exchange_strong(expected, fresh)) {
    cudaMemPoolDestroy(fresh);
    fresh = expected;
  }
  *out = fresh;
  return AA_OK;
}

// A library-owned non-blocking stream per device (the second stream of the
// host-buffer pipeline), created on first use.
std::atomic<cudaStream_t> g_side_stream[kMaxDevices];

int side_stream(cudaStream_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return AA_ERR_UNSUPPORTED;
  cudaStream_t s = g_side_stream[dev].load(std::memory_order_acquire);
  if (s != nullptr) {
    *out = s;
    return AA_OK;
  }
  e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreateWithFlags");
  cudaStream_t expected = nullptr;
  if (!g_side_stream[dev].compare_exchange_strong(expected, s)) {
    cudaStreamDestroy(s);      // another thread won the race
    s = expected;
  }
  *out = s;
  return AA_OK;
}

int scratch_alloc(void** ptr, size_t bytes, cudaStream_t st) {
  cudaMemPool_t pool = nullptr;
  int rc = device_pool(&pool);
  if (rc != AA_OK) return rc;
  cudaError_t e = cudaMallocFromPoolAsync(ptr, bytes, pool, st);
  return e == cudaSuccess ? AA_OK : cuda_fail(e, "cudaMallocFromPoolAsync");
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Components of one agent bias (fp32 device pointers, any may be null):
// row [H][k][grid_h], col [H][k][grid_w], block [H][k][pool_h*pool_w].
struct AgentBiasRef {
  const float* row;
  const float* col;
  const float* block;
  bool any() const { return row || col || block; }
};

struct Problem {
  int B, H, N, d, k;
  int grid_h, grid_w, pool_h, pool_w;  // pool_h == 0: learnable agents
  float scale;
  int dtype;
  const AgentBiasRef* b1 = nullptr;    // agent bias of the aggregation (agents x tokens)
  const AgentBiasRef* b2 = nullptr;    // agent bias of the broadcast (tokens x agents)
  bool force_simt = false;             // plan the SIMT kernels whatever the dtype
  long long BH() const { return (long long)B * H; }
  size_t elem() const { return dtype == AA_FP32 ? 4 : 2; }
};

int validate_common(int B, int H, int N, int d, int k, float scale, int dtype) {
  if (dtype != AA_FP32 && dtype != AA_BF16) return AA_ERR_UNSUPPORTED;
  if (B < 1 || H < 1 || N < 1) return AA_ERR_SHAPE;
  if (d < 8 || d > 128 || (d % 8) != 0) return AA_ERR_UNSUPPORTED;
  if (k < 1 || k > 256) return AA_ERR_UNSUPPORTED;
  if (!std::isfinite(scale) || !(scale > 0.f)) return AA_ERR_VALUE;
  if ((long long)B * H * (long long)N > (1LL << 40)) return AA_ERR_SHAPE;
  return AA_OK;
}

int validate_grid(int N, int grid_h, int grid_w, int pool_h, int pool_w) {
  if (grid_h < 1 || grid_w < 1 || (long long)grid_h * grid_w != N) return AA_ERR_SHAPE;
  if (pool_h < 1 || pool_w < 1 || pool_h > grid_h || pool_w > grid_w) return AA_ERR_SHAPE;
  return AA_OK;
}

bool has_bias(const Problem& p) { return (p.b1 && p.b1->any()) || (p.b2 && p.b2->any()); }
// Shared memory of the dense-copy builder (it builds B1, and B2 before its
// transpose): one agent row's row, column and block terms and the grid's cell
// tables, the per-axis arrays padded to 4 entries.
__host__ __device__ inline size_t bias_tokens_smem_bytes(int gh, int gw, int ph, int pw) {
  const size_t gh4 = ((size_t)gh + 3) & ~(size_t)3, gw4 = ((size_t)gw + 3) & ~(size_t)3;
  return sizeof(float) * (2 * (gh4 + gw4) + (size_t)ph * pw);
}
constexpr size_t kBiasSmemMax = 160 * 1024;
// The tensor-core kernels take the agent bias through dense copies while the
// builder's tables fit in shared memory (grid_h + grid_w up to about 20000);
// larger grids run the biased problem on the SIMT kernels.
bool use_tensor_cores(const Problem& p) {
  if (p.force_simt || p.dtype != AA_BF16 || !tc_supported(p.d, p.k)) return false;
  return !has_bias(p) ||
         bias_tokens_smem_bytes(p.grid_h, p.grid_w, p.pool_h, p.pool_w) <= kBiasSmemMax;
}

// Row lengths of the tensor-core kernels' dense bias copies: B1 [H][k][ld]
// (tokens, 16-byte rows), B2 [H][N][ld] (agents, k rounded up to 16).
int bias_ld_b1(const Problem& p) { return (p.N + 7) & ~7; }
int bias_ld_b2(const Problem& p) { return (p.k + 15) & ~15; }

void set_bias(SimtAttendArgs& a, const Problem& p, const AgentBiasRef* b, bool tok_is_col) {
  if (!b || !b->any()) return;
  a.bias_row = b->row;
  a.bias_col = b->col;
  a.bias_block = b->block;
  a.bias_tok_is_col = tok_is_col ? 1 : 0;
  a.grid_h = p.grid_h;
  a.grid_w = p.grid_w;
  a.pool_h = p.pool_h;
  a.pool_w = p.pool_w;
  a.n_agents = p.k;
}

// Scratch layout.  Every region starts on a 256-byte boundary.
struct Scratch {
  size_t a_off, va_off, pu_off, pml_off, total;
  size_t b1d_off, b2d_off;   // dense fp16 copies of B1 and B2 (tensor-core bias)
  size_t b2t_off;            // B2's tokens-contiguous copy, before its transpose
  SplitPlan plan;
  int simt_row_blocks;
  int simt_cols_per_split;
};

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

void plan_scratch(const Problem& p, int sm_count, Scratch* s) {
  const long long BH = p.BH();
  memset(s, 0, sizeof(*s));
  if (use_tensor_cores(p)) {
    tc_plan_aggregate(BH, p.N, p.k, sm_count, &s->plan);
  } else {
    const int row_blocks = (p.k + kSimtRows - 1) / kSimtRows;
    long long want = (2LL * sm_count + BH * row_blocks - 1) / (BH * row_blocks);
    const long long max_splits = (p.N + 127) / 128;
    if (want > max_splits) want = max_splits;
    if (want < 1) want = 1;
    int cps = (int)((p.N + want - 1) / want);
    cps = (cps + kSimtCols - 1) / kSimtCols * kSimtCols;
    const int splits = (p.N + cps - 1) / cps;
    s->plan.fixed = splits;
    s->plan.slots = splits;
    s->simt_row_blocks = row_blocks;
    s->simt_cols_per_split = cps;
  }
  const size_t agents_bytes = (size_t)BH * p.k * p.d * p.elem();
  size_t off = 0;
  s->a_off = off;
  off += round256(agents_bytes);
  s->va_off = off;
  off += round256(agents_bytes);
  s->pu_off = off;
  off += round256((size_t)BH * s->plan.slots * p.k * p.d * sizeof(float));
  s->pml_off = off;
  off += round256((size_t)BH * s->plan.slots * p.k * 2 * sizeof(float));
  s->b1d_off = off;
  if (use_tensor_cores(p) && p.b1 && p.b1->any())
    off += round256((size_t)p.H * p.k * bias_ld_b1(p) * sizeof(__half));
  s->b2d_off = off;
  if (use_tensor_cores(p) && p.b2 && p.b2->any())
    off += round256((size_t)p.H * p.N * bias_ld_b2(p) * sizeof(__half));
  s->b2t_off = off;
  if (use_tensor_cores(p) && p.b2 && p.b2->any())
    off += round256((size_t)p.H * p.k * bias_ld_b1(p) * sizeof(__half));
  s->total = off;
}

// Dense agent bias for the tensor-core kernels: (row + col + block) * log2(e)
// as fp16, saturated to the largest finite value, for agent a and grid token
// n = (y, x) of head h, the block term from the floor-partition cell
// (floor(y pool_h / grid_h), floor(x pool_w / grid_w)).
//   bias_dense_tokens_kernel: B1 [H][k][ld] (ld >= N, zero for n >= N);
//   B2 [H][N][ld] (ld = k rounded up to 16, zero for a >= k): the same
//   builder into scratch, then bias_transpose_kernel.
// Both read the components along their token axis (coalesced) and write
// whole rows of the dense copy.  fits32: every index product (grid side x
// pool side, the thread count) is below 2^31, so 32-bit divisions suffice.
__device__ __forceinline__ float bias_sum(const AgentBiasRef& b, long long ha, int y, int x,
                                          long long cell, int gh, int gw, long long n_cells) {
  float s = 0.f;
  if (b.row) s += __ldg(b.row + ha * gh + y);
  if (b.col) s += __ldg(b.col + ha * gw + x);
  if (b.block) s += __ldg(b.block + ha * n_cells + cell);
  return s;
}
__device__ __forceinline__ float bias_logit(float v) {
  return fminf(fmaxf(v * kLog2e, -65504.f), 65504.f);
}

__device__ __forceinline__ long long floor_div(long long a, int b, bool fits32) {
  return fits32 ? (long long)((int)a / b) : a / b;
}

// Block per agent row r = h k + a (grid-stride over the rows), 256 threads:
// the row's components (row terms [grid_h], column terms [grid_w], block
// terms [pool_h * pool_w]) are staged in shared memory beside the cell
// tables (cell row offset cy * pool_w per grid row, cell column per grid
// column); each thread then writes runs of 8 tokens as one 16-byte store.
// With grid_w a multiple of 8 a run lies in one grid row: its column terms
// and cell columns come as two 16-byte shared words each; otherwise each
// token finds its (y, x) by a division.
__global__ void __launch_bounds__(256) bias_dense_tokens_kernel(AgentBiasRef b,
                                                                __half* __restrict__ out, int H,
                                                                int k, int N, int gh, int gw,
                                                                int ph, int pw, int ld,
                                                                bool fits32) {
  extern __shared__ __align__(16) float bsm[];
  const int n_cells = ph * pw;
  const int gh4 = (gh + 3) & ~3, gw4 = (gw + 3) & ~3;
  float* s_row = bsm;                                   // [gh4]
  float* s_col = s_row + gh4;                           // [gw4], 16-byte aligned
  int* s_cx = reinterpret_cast<int*>(s_col + gw4);      // [gw4], 16-byte aligned
  int* s_cyo = s_cx + gw4;                              // [gh4]
  float* s_blk = reinterpret_cast<float*>(s_cyo + gh4); // [n_cells]
  const int tid = threadIdx.x;
  for (int i = tid; i < gh; i += blockDim.x)
    s_cyo[i] = (int)floor_div((long long)i * ph, gh, fits32) * pw;
  for (int i = tid; i < gw; i += blockDim.x) s_cx[i] = (int)floor_div((long long)i * pw, gw, fits32);
  const bool runs = (gw & 7) == 0;
  const long long rows = (long long)H * k;
  for (long long r = blockIdx.x; r < rows; r += gridDim.x) {
    __syncthreads();                         // the previous row's terms are read
    for (int i = tid; i < gh; i += blockDim.x) s_row[i] = b.row ? __ldg(b.row + r * gh + i) : 0.f;
    for (int i = tid; i < gw; i += blockDim.x) s_col[i] = b.col ? __ldg(b.col + r * gw + i) : 0.f;
    for (int i = tid; i < n_cells; i += blockDim.x)
      s_blk[i] = b.block ? __ldg(b.block + r * n_cells + i) : 0.f;
    __syncthreads();
    for (int c0 = 8 * tid; c0 < ld; c0 += 8 * blockDim.x) {
      float v[8];
      if (runs) {                            // N = grid_h grid_w is a multiple of 8 too
        if (c0 < N) {
          const int y = c0 / gw, x = c0 - y * gw;
          const float rw = s_row[y];
          const int cy = s_cyo[y];
          const float4 ca = *reinterpret_cast<const float4*>(s_col + x);
          const float4 cb = *reinterpret_cast<const float4*>(s_col + x + 4);
          const int4 xa = *reinterpret_cast<const int4*>(s_cx + x);
          const int4 xb = *reinterpret_cast<const int4*>(s_cx + x + 4);
          v[0] = rw + ca.x + s_blk[cy + xa.x];
          v[1] = rw + ca.y + s_blk[cy + xa.y];
          v[2] = rw + ca.z + s_blk[cy + xa.z];
          v[3] = rw + ca.w + s_blk[cy + xa.w];
          v[4] = rw + cb.x + s_blk[cy + xb.x];
          v[5] = rw + cb.y + s_blk[cy + xb.y];
          v[6] = rw + cb.z + s_blk[cy + xb.z];
          v[7] = rw + cb.w + s_blk[cy + xb.w];
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int n = c0 + e;
          v[e] = 0.f;
          if (n < N) {
            const int y = n / gw, x = n - y * gw;
            v[e] = s_row[y] + s_col[x] + s_blk[s_cyo[y] + s_cx[x]];
          }
        }
      }
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __half2 h2 = __floats2half2_rn(bias_logit(v[2 * e]), bias_logit(v[2 * e + 1]));
        memcpy(&w[e], &h2, sizeof(uint32_t));
      }
      *reinterpret_cast<uint4*>(out + r * ld + c0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// B2 in the agents-contiguous layout from its tokens-contiguous copy (built
// by bias_dense_tokens_kernel into scratch): src [H][k][lds] -> dst
// [H][N][ldd], zero for agents k .. ldd.  Block per (64 tokens, 64 agents,
// head), 256 threads.  Each thread loads 8 tokens of one agent as one 16-byte
// word and scatters them into a token-major tile (rows of 66 halves, 33
// words), then gathers 8 agents of one token as four 32-bit words (a warp's
// reads hit 32 banks) and stores them as one 16-byte word.
constexpr int kBiasT = 64;
constexpr int kBiasTRow = kBiasT + 2;               // halves per tile row
__global__ void __launch_bounds__(256) bias_transpose_kernel(const __half* __restrict__ src,
                                                             __half* __restrict__ dst, int k,
                                                             int N, int lds, int ldd) {
  __shared__ __align__(16) __half tile[kBiasT * kBiasTRow];   // [token][agent]
  const int n0 = blockIdx.x * kBiasT, a0 = blockIdx.y * kBiasT;
  const long long h = blockIdx.z;
  for (int i = threadIdx.x; i < kBiasT * (kBiasT / 8); i += blockDim.x) {
    const int a = i / (kBiasT / 8), p = i - a * (kBiasT / 8);
    const int n = n0 + 8 * p;                           // n < N: the 8 tokens lie in the row
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (a0 + a < k && n < N)
      w = *reinterpret_cast<const uint4*>(src + (h * k + a0 + a) * lds + n);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      tile[(8 * p + 2 * e) * kBiasTRow + a] = __ushort_as_half((unsigned short)(u[e] & 0xffffu));
      tile[(8 * p + 2 * e + 1) * kBiasTRow + a] = __ushort_as_half((unsigned short)(u[e] >> 16));
    }
  }
  __syncthreads();
  const uint32_t* t32 = reinterpret_cast<const uint32_t*>(tile);
  for (int i = threadIdx.x; i < kBiasT * (kBiasT / 8); i += blockDim.x) {
    const int jn = i / (kBiasT / 8), q = i - jn * (kBiasT / 8);
    const int n = n0 + jn, a = a0 + 8 * q;
    if (n >= N || a >= ldd) continue;
    const uint32_t* r = t32 + jn * (kBiasTRow / 2) + 4 * q;
    *reinterpret_cast<uint4*>(dst + (h * N + n) * ldd + a) = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

std::mutex g_smem_attr_mutex;   // serialises raising a kernel's shared-memory limit

template <typename KernelT>
int ensure_smem(KernelT kernel, size_t bytes, std::atomic<int>* flags) {
  int dev = 0;
  AA_CUDA(cudaGetDevice(&dev));
  if (dev < kMaxDevices && flags[dev].load(std::memory_order_acquire) >= (int)bytes)
    return AA_OK;
  // Check, raise and record under one lock, so that a smaller request of
  // another thread can never lower the limit after a larger one was recorded.
  std::lock_guard<std::mutex> lock(g_smem_attr_mutex);
  if (dev < kMaxDevices && flags[dev].load(std::memory_order_relaxed) >= (int)bytes)
    return AA_OK;
  AA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  if (dev < kMaxDevices) flags[dev].store((int)bytes, std::memory_order_release);
  return AA_OK;
}

std::atomic<int> g_simt_smem_f32[kMaxDevices];
std::atomic<int> g_simt_smem_bf16[kMaxDevices];

struct AgentsRef {
  const void* ptr;
  long long bstride, hstride;  // elements
};

std::atomic<int> g_pool_tma_smem_f32[kMaxDevices], g_pool_tma_smem_bf16[kMaxDevices];

template <typename T>
int launch_pool(const Problem& p, const void* q, float* a_f32, T* a_lowp, cudaStream_t st) {
  const PoolBandPlan bp = pool_band_plan(p.grid_h, p.grid_w, p.pool_h, p.pool_w, p.d);
  if (sizeof(T) == 2 && bp.ok) {
    const long long grid_x = (long long)p.pool_h * (p.pool_w / bp.bins);
    if (grid_x > 0x7fffffffLL) return AA_ERR_SHAPE;
    for (long long b0 = 0; b0 < p.BH(); b0 += 65535) {   // grid.y limit: slices in chunks
      const long long nb = (p.BH() - b0 < 65535) ? p.BH() - b0 : 65535;
      const long long qoff = b0 * (long long)p.N * p.d;
      const long long aoff = b0 * (long long)p.k * p.d;
      auto kernel = pool_band_batch(bp.rows_max) == 4 ? agent_pool_band_kernel<T, 4>
                                                      : agent_pool_band_kernel<T, kPoolBandBatch>;
      kernel<<<dim3((unsigned)grid_x, (unsigned)nb), bp.threads, bp.smem, st>>>(
          static_cast<const __nv_bfloat16*>(q) + qoff, a_f32 ? a_f32 + aoff : nullptr,
          a_lowp ? a_lowp + aoff : nullptr, p.N, p.d, p.grid_h, p.grid_w, p.pool_h, p.pool_w,
          bp.bins);
      AA_CUDA(cudaGetLastError());
    }
    return AA_OK;
  }
  const PoolTmaPlan tp = pool_tma_plan(p.grid_h, p.grid_w, p.pool_h, p.pool_w, p.d, (int)sizeof(T));
  if (tp.ok) {
    int rc = ensure_smem(agent_pool_tma_kernel<T>, tp.smem,
                         sizeof(T) == 4 ? g_pool_tma_smem_f32 : g_pool_tma_smem_bf16);
    if (rc != AA_OK) return rc;
    const int n_chunks = (p.pool_w + tp.px_per_cta - 1) / tp.px_per_cta;
    const long long grid_x = (long long)p.pool_h * n_chunks;
    if (grid_x > 0x7fffffffLL) return AA_ERR_SHAPE;
    const int tile_region =
        (int)((((size_t)tp.rows_max * tp.cols_max * p.d * sizeof(T)) + 127) & ~(size_t)127);
    for (long long b0 = 0; b0 < p.BH(); b0 += 65535) {   // grid.y limit: slices in chunks
      const long long nb = (p.BH() - b0 < 65535) ? p.BH() - b0 : 65535;
      const long long qoff = b0 * (long long)p.N * p.d;
      const long long aoff = b0 * (long long)p.k * p.d;
      agent_pool_tma_kernel<T><<<dim3((unsigned)grid_x, (unsigned)nb), kPoolTmaThreads, tp.smem,
                                 st>>>(
          static_cast<const T*>(q) + qoff, a_f32 ? a_f32 + aoff : nullptr,
          a_lowp ? a_lowp + aoff : nullptr, p.N, p.d, p.grid_h, p.grid_w, p.pool_h, p.pool_w,
          tp.px_per_cta, tp.cols_max, tile_region);
      AA_CUDA(cudaGetLastError());
    }
    return AA_OK;
  }
  const int per = pool_px_per_cta(p.grid_w, p.pool_w, p.d);
  const int n_chunks = (p.pool_w + per - 1) / per;
  const int groups = p.d / 8;
  // token columns a chunk can span: per bins, each at most ceil(G/P) + 1 wide,
  // processed in windows of pool_window_cols columns
  int cols = per * ((p.grid_w + p.pool_w - 1) / p.pool_w + 1);
  if (cols > pool_window_cols(p.d)) cols = pool_window_cols(p.d);
  const size_t smem = (size_t)cols * groups * 8 * sizeof(float);
  static std::atomic<int> flags[kMaxDevices];
  int rc = ensure_smem(agent_pool_kernel<T>, smem, flags);
  if (rc != AA_OK) return rc;
  const long long grid_x = (long long)p.pool_h * n_chunks;
  if (grid_x > 0x7fffffffLL) return AA_ERR_SHAPE;
  for (long long b0 = 0; b0 < p.BH(); b0 += 65535) {     // grid.y limit: slices in chunks
    const long long nb = (p.BH() - b0 < 65535) ? p.BH() - b0 : 65535;
    const long long qoff = b0 * (long long)p.N * p.d;
    const long long aoff = b0 * (long long)p.k * p.d;
    agent_pool_kernel<T><<<dim3((unsigned)grid_x, (unsigned)nb), kPoolThreads, smem, st>>>(
        static_cast<const T*>(q) + qoff, a_f32 ? a_f32 + aoff : nullptr,
        a_lowp ? a_lowp + aoff : nullptr, p.N, p.d, p.grid_h, p.grid_w, p.pool_h, p.pool_w, per);
    AA_CUDA(cudaGetLastError());
  }
  return AA_OK;
}

template <typename T>
int launch_simt_attend(const SimtAttendArgs& args, long long BH, cudaStream_t st, bool pdl) {
  const size_t smem = simt_attend_smem_bytes(args.d);
  int rc = ensure_smem(simt_attend_kernel<T>, smem,
                       sizeof(T) == 4 ? g_simt_smem_f32 : g_simt_smem_bf16);
  if (rc != AA_OK) return rc;
  const long long blocks = BH * args.splits * args.row_blocks;
  if (blocks > 0x7fffffffLL) return AA_ERR_SHAPE;
  AA_CUDA(launch_kernel(simt_attend_kernel<T>, dim3((unsigned)blocks), dim3(kSimtThreads), smem, st,
                        pdl, args));
  return AA_OK;
}

std::atomic<int> g_bias_tokens_smem[kMaxDevices];

// B1 (tokens_minor) straight into `out`; B2 through `tmp` (a tokens-contiguous
// copy of H k (N rounded up to 8) halves).
int launch_bias_dense(const Problem& p, const AgentBiasRef& b, __half* out, bool tokens_minor,
                      cudaStream_t st, __half* tmp) {
  const long long lim = 0x7fffffffLL;
  bool fits32 = (long long)p.grid_h * p.pool_h <= lim && (long long)p.grid_w * p.pool_w <= lim;
  if (tokens_minor) {
    const size_t smem = bias_tokens_smem_bytes(p.grid_h, p.grid_w, p.pool_h, p.pool_w);
    int rc = ensure_smem(bias_dense_tokens_kernel, smem, g_bias_tokens_smem);
    if (rc != AA_OK) return rc;
    const long long rows = (long long)p.H * p.k;
    bias_dense_tokens_kernel<<<(unsigned)(rows < 65535 ? rows : 65535), 256, smem, st>>>(
        b, out, p.H, p.k, p.N, p.grid_h, p.grid_w, p.pool_h, p.pool_w, bias_ld_b1(p), fits32);
  } else {
    // tokens-contiguous into `tmp`, then transposed into `out`
    if (tmp == nullptr) return AA_ERR_WORKSPACE;
    int rc = launch_bias_dense(p, b, tmp, true, st, nullptr);
    if (rc != AA_OK) return rc;
    const int ldd = bias_ld_b2(p);
    const dim3 grid((unsigned)((p.N + kBiasT - 1) / kBiasT), (unsigned)((ldd + kBiasT - 1) / kBiasT),
                    (unsigned)p.H);
    if (p.H > 65535) return AA_ERR_SHAPE;
    bias_transpose_kernel<<<grid, 256, 0, st>>>(tmp, out, p.k, p.N, bias_ld_b1(p), ldd);
  }
  AA_CUDA(cudaGetLastError());
  return AA_OK;
}

template <typename T>
int launch_merge(const Problem& p, const Scratch& s, char* ws, float* va_f32, T* va_lowp,
                 cudaStream_t st, bool pdl, float* ml_out = nullptr) {
  const long long work = p.BH() * p.k * (p.d / 4);
  const long long blocks = (work + kMergeThreads - 1) / kMergeThreads;
  if (blocks > 0x7fffffffLL) return AA_ERR_SHAPE;
  AA_CUDA(launch_kernel(agent_merge_kernel<T>, dim3((unsigned)blocks), dim3(kMergeThreads), 0, st,
                        pdl, reinterpret_cast<const float*>(ws + s.pu_off),
                        reinterpret_cast<const float*>(ws + s.pml_off), s.plan, p.BH(), p.k, p.d,
                        va_f32, va_lowp, ml_out));
  return AA_OK;
}

// Aggregation + merge.  agents are in the run dtype (fp32 path: float).  With
// pdl, the aggregation overlaps the tail of the previous kernel of the stream.
template <typename T>
int run_aggregate(const Problem& p, const Scratch& s, const AgentsRef& ag, const void* k,
                  const void* v, char* ws, float* va_f32, T* va_lowp, cudaStream_t st,
                  bool pdl = false) {
  const long long qstride_h = (long long)p.N * p.d, qstride_b = qstride_h * p.H;
  if (use_tensor_cores(p)) {
    tc::BiasParams b1{nullptr, 0};
    if (p.b1 && p.b1->any())
      b1 = tc::BiasParams{reinterpret_cast<const __half*>(ws + s.b1d_off), bias_ld_b1(p)};
    cudaError_t e = tc_launch_aggregate(ag.ptr, ag.bstride, ag.hstride, k, v, p.B, p.H, p.N, p.d,
                                        p.k, p.scale * kLog2e, s.plan,
                                        reinterpret_cast<float*>(ws + s.pu_off),
                                        reinterpret_cast<float*>(ws + s.pml_off), st, pdl, &b1);
    if (e != cudaSuccess) return cuda_fail(e, "agent_aggregate (tensor cores) launch");
  } else {
    SimtAttendArgs a;
    memset(&a, 0, sizeof(a));
    a.rows = ag.ptr;
    a.rows_bstride = ag.bstride;
    a.rows_hstride = ag.hstride;
    a.cols = k;
    a.cols_bstride = qstride_b;
    a.cols_hstride = qstride_h;
    a.vals = v;
    a.vals_bstride = qstride_b;
    a.vals_hstride = qstride_h;
    a.H = p.H;
    a.n_rows = p.k;
    a.n_cols = p.N;
    a.d = p.d;
    a.scale_log2 = p.scale * kLog2e;
    a.row_blocks = s.simt_row_blocks;
    a.splits = s.plan.fixed;
    a.cols_per_split = s.simt_cols_per_split;
    a.part_u = reinterpret_cast<float*>(ws + s.pu_off);
    a.part_ml = reinterpret_cast<float*>(ws + s.pml_off);
    a.slots = s.plan.slots;
    set_bias(a, p, p.b1, true);
    int rc = launch_simt_attend<T>(a, p.BH(), st, pdl);
    if (rc != AA_OK) return rc;
  }
  return launch_merge<T>(p, s, ws, va_f32, va_lowp, st, true);
}

template <typename T>
int run_broadcast(const Problem& p, const void* q, const AgentsRef& ag, const void* va,
                  void* out, cudaStream_t st, bool pdl = false,
                  const __half* b2d = nullptr) {
  const long long qstride_h = (long long)p.N * p.d, qstride_b = qstride_h * p.H;
  const long long vstride_h = (long long)p.k * p.d, vstride_b = vstride_h * p.H;
  if (use_tensor_cores(p)) {
    int sms = 0;
    int rc = device_sm_count(&sms);
    if (rc != AA_OK) return rc;
    tc::BiasParams b2{nullptr, 0};
    if (p.b2 && p.b2->any()) {
      if (b2d == nullptr) return AA_ERR_WORKSPACE;
      b2 = tc::BiasParams{b2d, bias_ld_b2(p)};
    }
    cudaError_t e = tc_launch_broadcast(q, ag.ptr, ag.bstride, va, out, p.B, p.H, p.N, p.d, p.k,
                                        p.scale * kLog2e, sms, st, pdl, &b2);
    if (e != cudaSuccess) return cuda_fail(e, "agent_broadcast (tensor cores) launch");
    return AA_OK;
  }
  SimtAttendArgs a;
  memset(&a, 0, sizeof(a));
  a.rows = q;
  a.rows_bstride = qstride_b;
  a.rows_hstride = qstride_h;
  a.cols = ag.ptr;
  a.cols_bstride = ag.bstride;
  a.cols_hstride = ag.hstride;
  a.vals = va;
  a.vals_bstride = vstride_b;
  a.vals_hstride = vstride_h;
  a.H = p.H;
  a.n_rows = p.N;
  a.n_cols = p.k;
  a.d = p.d;
  a.scale_log2 = p.scale * kLog2e;
  a.row_blocks = (p.N + kSimtRows - 1) / kSimtRows;
  a.splits = 1;
  a.cols_per_split = p.k;
  a.out = out;
  a.out_bstride = qstride_b;
  a.out_hstride = qstride_h;
  set_bias(a, p, p.b2, false);
  return launch_simt_attend<T>(a, p.BH(), st, pdl);
}

// Small bf16 slices (pooled or given agents, no bias) run the whole pass in
// one kernel, one CTA per slice (agent_fused_small_tc).
bool use_fused_small(const Problem& p) {
  return !p.force_simt && p.dtype == AA_BF16 && !has_bias(p) &&
         tc::fused_small_fits(p.N, p.d, p.k);
}

template <typename T>
int run_forward(const Problem& p, const Scratch& s, const void* q, const void* k, const void* v,
                const AgentsRef* learnable, void* out, char* ws, cudaStream_t st) {
  if (sizeof(T) == 2 && use_fused_small(p)) {
    cudaError_t e = tc_launch_fused_small(
        q, k, v, out, p.B, p.H, p.N, p.d, p.grid_h, p.grid_w, p.pool_h, p.pool_w, p.k,
        learnable ? learnable->ptr : nullptr, learnable ? learnable->bstride : 0,
        p.scale * kLog2e, st);
    if (e != cudaSuccess) return cuda_fail(e, "agent forward (fused small slices) launch");
    return AA_OK;
  }
  if (use_tensor_cores(p)) {
    // the dense bias copies, before the pool: every later kernel of the pass
    // starts after they have completed (the pool launches without overlap)
    if (p.b1 && p.b1->any()) {
      int rc = launch_bias_dense(p, *p.b1, reinterpret_cast<__half*>(ws + s.b1d_off), true, st,
                                 nullptr);
      if (rc != AA_OK) return rc;
    }
    if (p.b2 && p.b2->any()) {
      int rc = launch_bias_dense(p, *p.b2, reinterpret_cast<__half*>(ws + s.b2d_off), false, st,
                                 reinterpret_cast<__half*>(ws + s.b2t_off));
      if (rc != AA_OK) return rc;
    }
  }
  AgentsRef ag;
  const long long ahs = (long long)p.k * p.d;
  if (learnable) {
    ag = *learnable;
  } else {
    T* a_ws = reinterpret_cast<T*>(ws + s.a_off);
    int rc = (sizeof(T) == 4)
                 ? launch_pool<T>(p, q, reinterpret_cast<float*>(a_ws), nullptr, st)
                 : launch_pool<T>(p, q, nullptr, a_ws, st);
    if (rc != AA_OK) return rc;
    ag.ptr = a_ws;
    ag.bstride = ahs * p.H;
    ag.hstride = ahs;
  }
  // The pool launches normally (it follows whatever the stream did before);
  // the kernels after it overlap their predecessors' tails (programmatic
  // dependent launch) and read their outputs only after a grid dependency wait.
  const bool pdl_agg = learnable == nullptr;
  T* va_ws = reinterpret_cast<T*>(ws + s.va_off);
  int rc = (sizeof(T) == 4)
               ? run_aggregate<T>(p, s, ag, k, v, ws, reinterpret_cast<float*>(va_ws), nullptr,
                                  st, pdl_agg)
               : run_aggregate<T>(p, s, ag, k, v, ws, nullptr, va_ws, st, pdl_agg);
  if (rc != AA_OK) return rc;
  return run_broadcast<T>(p, q, ag, va_ws, out, st, true,
                          reinterpret_cast<const __half*>(ws + s.b2d_off));
}

int forward_impl(const Problem& p, const void* q, const void* k, const void* v,
                 const AgentsRef* learnable, void* out, void* user_ws, size_t user_ws_bytes,
                 bool have_user_ws, cudaStream_t st) {
  int sms = 0;
  int rc = device_sm_count(&sms);
  if (rc != AA_OK) return rc;
  Scratch s;
  plan_scratch(p, sms, &s);
  char* ws = nullptr;
  bool owned = false;
  if (have_user_ws) {
    if (user_ws == nullptr) return AA_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(user_ws) & 255u) != 0) return AA_ERR_ALIGN;
    if (user_ws_bytes < s.total) return AA_ERR_WORKSPACE;
    ws = static_cast<char*>(user_ws);
  } else {
    rc = scratch_alloc(reinterpret_cast<void**>(&ws), s.total, st);
    if (rc != AA_OK) return rc;
    owned = true;
  }
  rc = (p.dtype == AA_FP32)
           ? run_forward<float>(p, s, q, k, v, learnable, out, ws, st)
           : run_forward<__nv_bfloat16>(p, s, q, k, v, learnable, out, ws, st);
  if (owned) {
    cudaError_t e = cudaFreeAsync(ws, st);
    if (rc == AA_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  }
  return rc;
}

int check_tensor_ptrs(const void* q, const void* k, const void* v, const void* out) {
  if (!q || !k || !v || !out) return AA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return AA_ERR_ALIGN;
  return AA_OK;
}

int pooled_forward(const void* q, const void* k, const void* v, const void* agents_or_null,
                   void* out, int B, int H, int N, int d, int grid_h, int grid_w, int pool_h,
                   int pool_w, float scale, int dtype, void* ws, size_t ws_bytes, bool have_ws,
                   void* stream) {
  int rc = validate_grid(N, grid_h, grid_w, pool_h, pool_w);
  if (rc != AA_OK) return rc;
  const int kk = pool_h * pool_w;
  rc = validate_common(B, H, N, d, kk, scale, dtype);
  if (rc != AA_OK) return rc;
  rc = check_tensor_ptrs(q, k, v, out);
  if (rc != AA_OK) return rc;
  if (agents_or_null && !aligned16(agents_or_null)) return AA_ERR_ALIGN;
  Problem p{B, H, N, d, kk, grid_h, grid_w, pool_h, pool_w, scale, dtype};
  AgentsRef learn{agents_or_null, 0, (long long)kk * d};
  return forward_impl(p, q, k, v, agents_or_null ? &learn : nullptr, out, ws, ws_bytes, have_ws,
                      static_cast<cudaStream_t>(stream));
}

// Depth-wise 3x3 term: out (+)= DWConv3x3(v) over the grid, per (head, channel).
std::atomic<int> g_dwc_stream_f32[kMaxDevices], g_dwc_stream_bf16[kMaxDevices];

template <typename T>
int dwc_stream_launch(const void* v, const float* w, const float* bias, void* out, int H,
                      int grid_h, int grid_w, int d, int accumulate, long long BH,
                      const DwcStreamPlan& pl, int sms, cudaStream_t st, bool pdl) {
  int rc = ensure_smem(dwc_stream_kernel<T>, pl.smem,
                       sizeof(T) == 4 ? g_dwc_stream_f32 : g_dwc_stream_bf16);
  if (rc != AA_OK) return rc;
  int per_sm = 0;
  AA_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dwc_stream_kernel<T>,
                                                        pl.threads, pl.smem));
  if (per_sm < 1) return AA_ERR_SHAPE;
  const int band = dwc_stream_band(grid_h, BH * pl.n_xc, (long long)sms * per_sm);
  const long long grid_x = (long long)((grid_h + band - 1) / band) * pl.n_xc;
  if (grid_x > 0x7fffffffLL || BH > 65535) return AA_ERR_SHAPE;
  AA_CUDA(launch_kernel(dwc_stream_kernel<T>, dim3((unsigned)grid_x, (unsigned)BH),
                        dim3(pl.threads), pl.smem, st, pdl, static_cast<const T*>(v), w, bias,
                        static_cast<T*>(out), H, grid_h, grid_w, d, pl.cols, band, pl.vslot,
                        accumulate));
  return AA_OK;
}

int dwc_impl(const void* v, const float* w, const float* bias, void* out, int B, int H,
             int grid_h, int grid_w, int d, int dtype, int accumulate, cudaStream_t st, bool pdl) {
  const long long BH = (long long)B * H;
  if (BH <= 65535) {
    int sms = 0;
    int rc = device_sm_count(&sms);
    if (rc != AA_OK) return rc;
    const DwcStreamPlan pl = dwc_stream_plan(grid_w, d, dtype == AA_FP32 ? 4 : 2);
    if (pl.ok)
      return dtype == AA_FP32
                 ? dwc_stream_launch<float>(v, w, bias, out, H, grid_h, grid_w, d, accumulate,
                                            BH, pl, sms, st, pdl)
                 : dwc_stream_launch<__nv_bfloat16>(v, w, bias, out, H, grid_h, grid_w, d,
                                                    accumulate, BH, pl, sms, st, pdl);
  }
  const long long N = (long long)grid_h * grid_w;
  const long long items = (long long)grid_h * ((grid_w + kDwcSpan - 1) / kDwcSpan) * (d / 8);
  if (N * (d / 8) >= (1LL << 31)) return AA_ERR_SHAPE;   // checked by validate_dwc too
  const long long blocks = (items + kDwcThreads - 1) / kDwcThreads;
  const dim3 grid((unsigned)blocks, (unsigned)(BH < 65535 ? BH : 65535));
  const size_t smem = (size_t)10 * d * sizeof(float);
  cudaError_t e;
  if (dtype == AA_FP32)
    e = launch_kernel(dwc_kernel<float>, grid, dim3(kDwcThreads), smem, st, pdl,
                      static_cast<const float*>(v), w, bias, static_cast<float*>(out), H, grid_h,
                      grid_w, d, BH, accumulate);
  else
    e = launch_kernel(dwc_kernel<__nv_bfloat16>, grid, dim3(kDwcThreads), smem, st, pdl,
                      static_cast<const __nv_bfloat16*>(v), w, bias,
                      static_cast<__nv_bfloat16*>(out), H, grid_h, grid_w, d, BH, accumulate);
  if (e != cudaSuccess) return cuda_fail(e, "dwc_kernel launch");
  return AA_OK;
}

int validate_dwc(const void* v, const float* w, const void* out, int B, int H, int grid_h,
                 int grid_w, int d, int dtype) {
  if (dtype != AA_FP32 && dtype != AA_BF16) return AA_ERR_UNSUPPORTED;
  if (B < 1 || H < 1 || grid_h < 1 || grid_w < 1) return AA_ERR_SHAPE;
  if (d < 8 || d > 128 || (d % 8) != 0) return AA_ERR_UNSUPPORTED;
  if ((long long)B * H * grid_h * (long long)grid_w > (1LL << 40)) return AA_ERR_SHAPE;
  if ((long long)grid_h * grid_w * (d / 8) >= (1LL << 31)) return AA_ERR_SHAPE;
  if (!v || !w || !out) return AA_ERR_NULL;
  if (!aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(w) & 3u)) return AA_ERR_ALIGN;
  return AA_OK;
}

// ------------------------------------------------------------ backward pass
std::atomic<int> g_bwd_q_f32[kMaxDevices], g_bwd_q_bf16[kMaxDevices];
std::atomic<int> g_bwd_qr_f32[kMaxDevices], g_bwd_qr_bf16[kMaxDevices];
std::atomic<int> g_bwd_k_f32[kMaxDevices], g_bwd_k_bf16[kMaxDevices];
std::atomic<int> g_simt_f32rows_f32[kMaxDevices], g_simt_f32rows_bf16[kMaxDevices];

// Learnable agents [H][k][d] of T (shared over the batch) -> fp32 [BH][k][d].
template <typename T>
__global__ void expand_agents_f32_kernel(const T* __restrict__ ag, float* __restrict__ out,
                                         long long BH, int H, long long kd) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= BH * kd) return;
  const long long bh = e / kd, r = e - bh * kd;
  out[e] = to_f32(ag[(bh % H) * kd + r]);
}

// Steps 3-5 of the backward pass, given the fp32 agents, V_A and each agent
// row's softmax max and sum: the broadcast-stage gradients, the
// aggregation-stage gradients, then dQ with the pooling adjoint and the
// agents' own gradient.
// The tensor-core pass over K that gives the key kernel its exponentials:
// the bf16 agents and V_A the broadcast reads, and the SM count it sizes its
// grid by.
struct KeyExpLaunch {
  const void* agents;
  long long agents_bstride;
  const void* va_low;
  int sms;
};

template <typename T>
int backward_gradients(const Problem& p, const void* q, const void* k, const void* v,
                       const void* agents, const void* dout, void* dq, void* dk, void* dv,
                       float* dagents, float* a32, float* va32, float* ml, float* dva, float* da,
                       float* dqa, float* ej, cudaStream_t st,
                       const tc::BcStats* qstats = nullptr,
                       const KeyExpLaunch* kexp = nullptr) {
  const long long BH = p.BH();
  const size_t kd = (size_t)p.k * p.d;
  const size_t nd = (size_t)p.N * p.d;
  int r = AA_OK;
  // 3. broadcast-stage gradients
  AA_CUDA(cudaMemsetAsync(dva, 0, BH * kd * 4, st));
  AA_CUDA(cudaMemsetAsync(da, 0, BH * kd * 4, st));
  BwdArgs g;
  memset(&g, 0, sizeof(g));
  g.x = q;
  g.y = dout;
  g.a = a32;
  g.va = va32;
  g.dq = dqa;
  g.dva_acc = dva;
  g.da_acc = da;
  g.N = p.N;
  g.n_agents = p.k;
  g.d = p.d;
  g.scale = p.scale;
  g.scale_log2 = p.scale * kLog2e;
  if (qstats) {
    g.st_m = qstats->m;
    g.st_l = qstats->l;
    g.st_D = qstats->D;
    g.st_p = reinterpret_cast<const uint32_t*>(qstats->p);
    g.st_kpad = (p.k + 15) / 16 * 16;
  }
  const size_t smem_b = bwd_smem_bytes(p.d);
  const dim3 grid_b((unsigned)((p.N + kBwdRows - 1) / kBwdRows), (unsigned)BH);
  if (p.d <= 64) {   // dQ accumulated in registers: 16 (d / 4) <= 256 threads
    const size_t smem_q = bwd_query_reg_smem_bytes(p.d);
    r = ensure_smem(bwd_query_kernel<T, true>, smem_q,
                    sizeof(T) == 4 ? g_bwd_qr_f32 : g_bwd_qr_bf16);
    if (r != AA_OK) return r;
    bwd_query_kernel<T, true><<<grid_b, kBwdThreads, smem_q, st>>>(g);
  } else {
    r = ensure_smem(bwd_query_kernel<T>, smem_b, sizeof(T) == 4 ? g_bwd_q_f32 : g_bwd_q_bf16);
    if (r != AA_OK) return r;
    bwd_query_kernel<T><<<grid_b, kBwdThreads, smem_b, st>>>(g);
  }
  AA_CUDA(cudaGetLastError());
  // 4. aggregation-stage gradients, with E_j = dV_A_j . V_A_j computed once
  // per (slice, agent)
  {
    const long long rows = BH * (long long)p.k;
    bwd_agent_e_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(dva, va32, ej, rows,
                                                                           p.d);
    AA_CUDA(cudaGetLastError());
  }
  g.st_m = g.st_l = g.st_D = nullptr;
  g.st_p = nullptr;
  if (qstats && kexp) {
    // the broadcast over K in column mode: 2^(s - m_j) for every (key, agent
    // j), m_j the aggregation's max, into the buffer the query kernel has
    // finished with
    const tc::BcStats ks{nullptr, nullptr, nullptr, nullptr, qstats->p, ml};
    cudaError_t e = tc_launch_broadcast(k, kexp->agents, kexp->agents_bstride, kexp->va_low,
                                        const_cast<void*>(k), p.B, p.H, p.N, p.d, p.k,
                                        p.scale * kLog2e, kexp->sms, st, false, nullptr, &ks);
    if (e != cudaSuccess) return cuda_fail(e, "agent_broadcast (backward key exponentials) launch");
    g.st_p = reinterpret_cast<const uint32_t*>(qstats->p);
    g.st_kpad = (p.k + 15) / 16 * 16;
  }
  g.x = k;
  g.y = v;
  g.dva = dva;
  g.ml = ml;
  g.e = ej;
  g.dk = dk;
  g.dv = dv;
  r = ensure_smem(bwd_key_kernel<T>, smem_b, sizeof(T) == 4 ? g_bwd_k_f32 : g_bwd_k_bf16);
  if (r != AA_OK) return r;
  bwd_key_kernel<T><<<grid_b, kBwdThreads, smem_b, st>>>(g);
  AA_CUDA(cudaGetLastError());
  // 5. dQ (+ pooling adjoint) in the run dtype; the agents' own gradient
  const dim3 grid_f((unsigned)(((long long)nd / 8 + 255) / 256), (unsigned)BH);
  bwd_finish_kernel<T><<<grid_f, 256, 0, st>>>(dqa, da, static_cast<T*>(dq), p.N, p.d, p.grid_h,
                                               p.grid_w, p.pool_h, p.pool_w,
                                               agents == nullptr ? 1 : 0);
  AA_CUDA(cudaGetLastError());
  if (dagents) AA_CUDA(cudaMemcpyAsync(dagents, da, BH * kd * 4, cudaMemcpyDeviceToDevice, st));
  return AA_OK;
}

template <typename T>
int backward_impl(const Problem& p, const void* q, const void* k, const void* v,
                  const void* agents, const void* dout, void* dq, void* dk, void* dv,
                  float* dagents, cudaStream_t st) {
  int sms = 0;
  int rc = device_sm_count(&sms);
  if (rc != AA_OK) return rc;
  // bf16 with d <= 64: the forward statistics are recomputed on the tensor
  // cores from the bf16 agents the forward pass uses, and the gradient
  // kernels take the same bf16 agents widened to fp32, so the saved maxima
  // and sums match the scores they recompute; otherwise the SIMT aggregation
  // with fp32 agents.
  const bool tc_recompute = sizeof(T) == 2 && tc_supported(p.d, p.k);
  Problem pp = p;
  pp.force_simt = !tc_recompute;
  Scratch s;
  plan_scratch(pp, sms, &s);
  const long long BH = p.BH();
  const size_t kd = (size_t)p.k * p.d;
  const size_t nd = (size_t)p.N * p.d;
  // workspace: plan regions (partials) + fp32 agents, V_A, (max, sum), dV_A, dA, dQ
  size_t off = s.total;
  const size_t a32_off = off;   off += round256(BH * kd * 4);
  const size_t va32_off = off;  off += round256(BH * kd * 4);
  const size_t ml_off = off;    off += round256(BH * (size_t)p.k * 2 * 4);
  const size_t dva_off = off;   off += round256(BH * kd * 4);
  const size_t da_off = off;    off += round256(BH * kd * 4);
  const size_t dq_off = off;    off += round256(BH * nd * 4);
  const size_t e_off = off;     off += round256(BH * (size_t)p.k * 4);
  // the broadcast's per-query statistics (max, sum, D) and exponentials
  // 2^(s - m) (bf16, k padded to 16) from the tensor cores
  const size_t kpad16 = (size_t)(p.k + 15) / 16 * 16;
  const size_t st_off = off;    off += tc_recompute ? 3 * round256(BH * (size_t)p.N * 4) : 0;
  const size_t sp_off = off;    off += tc_recompute ? round256(BH * (size_t)p.N * kpad16 * 2) : 0;
  char* ws = nullptr;
  rc = scratch_alloc(reinterpret_cast<void**>(&ws), off, st);
  if (rc != AA_OK) return rc;
  float* a32 = reinterpret_cast<float*>(ws + a32_off);
  float* va32 = reinterpret_cast<float*>(ws + va32_off);
  float* ml = reinterpret_cast<float*>(ws + ml_off);
  float* dva = reinterpret_cast<float*>(ws + dva_off);
  float* da = reinterpret_cast<float*>(ws + da_off);
  float* dqa = reinterpret_cast<float*>(ws + dq_off);
  float* ej = reinterpret_cast<float*>(ws + e_off);
  auto run = [&]() -> int {
    const long long n_ag = BH * (long long)kd;
    if (tc_recompute) {
      // 1. bf16 agents (pooled, or the given ones) and their fp32 widening
      const void* ag = agents;
      long long ag_bstride = 0;
      if (agents == nullptr) {
        T* a_low = reinterpret_cast<T*>(ws + s.a_off);
        int r = launch_pool<T>(p, q, nullptr, a_low, st);
        if (r != AA_OK) return r;
        ag = a_low;
        ag_bstride = (long long)kd * p.H;
        expand_agents_f32_kernel<T><<<(unsigned)((n_ag + 255) / 256), 256, 0, st>>>(
            a_low, a32, BH, (int)BH, (long long)kd);
      } else {
        expand_agents_f32_kernel<T><<<(unsigned)((n_ag + 255) / 256), 256, 0, st>>>(
            static_cast<const T*>(agents), a32, BH, p.H, (long long)kd);
      }
      AA_CUDA(cudaGetLastError());
      // 2. forward aggregation on the tensor cores: V_A (fp32) and each agent
      // row's max and sum from the merge
      cudaError_t e = tc_launch_aggregate(ag, ag_bstride, (long long)kd, k, v, p.B, p.H, p.N, p.d,
                                          p.k, p.scale * kLog2e, s.plan,
                                          reinterpret_cast<float*>(ws + s.pu_off),
                                          reinterpret_cast<float*>(ws + s.pml_off), st, false);
      if (e != cudaSuccess) return cuda_fail(e, "agent_aggregate (backward recompute) launch");
      T* va_low = reinterpret_cast<T*>(ws + s.va_off);
      int r = launch_merge<T>(pp, s, ws, va32, va_low, st, false, ml);
      if (r != AA_OK) return r;
      // 3. the broadcast on the tensor cores, writing each query's max, sum,
      // D = dO . O and exponentials instead of O (the gradient kernel's first
      // sweep and its score dot products)
      const size_t st_bytes = round256(BH * (size_t)p.N * 4);
      const tc::BcStats qs{static_cast<const __nv_bfloat16*>(dout),
                           reinterpret_cast<float*>(ws + st_off),
                           reinterpret_cast<float*>(ws + st_off + st_bytes),
                           reinterpret_cast<float*>(ws + st_off + 2 * st_bytes),
                           reinterpret_cast<__nv_bfloat16*>(ws + sp_off)};
      e = tc_launch_broadcast(q, ag, ag_bstride, va_low, const_cast<void*>(q), p.B, p.H, p.N, p.d,
                              p.k, p.scale * kLog2e, sms, st, false, nullptr, &qs);
      if (e != cudaSuccess) return cuda_fail(e, "agent_broadcast (backward statistics) launch");
      const KeyExpLaunch kx{ag, ag_bstride, va_low, sms};
      return backward_gradients<T>(p, q, k, v, agents, dout, dq, dk, dv, dagents, a32, va32, ml,
                                   dva, da, dqa, ej, st, &qs, &kx);
    }
    // 1. fp32 agents
    if (agents == nullptr) {
      int r = launch_pool<T>(p, q, a32, nullptr, st);
      if (r != AA_OK) return r;
    } else {
      expand_agents_f32_kernel<T><<<(unsigned)((n_ag + 255) / 256), 256, 0, st>>>(
          static_cast<const T*>(agents), a32, BH, p.H, (long long)kd);
      AA_CUDA(cudaGetLastError());
    }
    // 2. forward aggregation with fp32 agent rows: V_A and each row's max and sum
    SimtAttendArgs a;
    memset(&a, 0, sizeof(a));
    const long long qstride_h = (long long)nd, qstride_b = qstride_h * p.H;
    a.rows = a32;
    a.rows_bstride = (long long)kd * p.H;
    a.rows_hstride = (long long)kd;
    a.cols = k;
    a.cols_bstride = qstride_b;
    a.cols_hstride = qstride_h;
    a.vals = v;
    a.vals_bstride = qstride_b;
    a.vals_hstride = qstride_h;
    a.H = p.H;
    a.n_rows = p.k;
    a.n_cols = p.N;
    a.d = p.d;
    a.scale_log2 = p.scale * kLog2e;
    a.row_blocks = s.simt_row_blocks;
    a.splits = s.plan.fixed;
    a.cols_per_split = s.simt_cols_per_split;
    a.part_u = reinterpret_cast<float*>(ws + s.pu_off);
    a.part_ml = reinterpret_cast<float*>(ws + s.pml_off);
    a.slots = s.plan.slots;
    const size_t smem_a = simt_attend_smem_bytes(p.d);
    int r = ensure_smem(simt_attend_kernel<T, float>, smem_a,
                        sizeof(T) == 4 ? g_simt_f32rows_f32 : g_simt_f32rows_bf16);
    if (r != AA_OK) return r;
    const long long blocks = BH * a.splits * a.row_blocks;
    if (blocks > 0x7fffffffLL) return AA_ERR_SHAPE;
    AA_CUDA(launch_kernel(simt_attend_kernel<T, float>, dim3((unsigned)blocks), dim3(kSimtThreads),
                          smem_a, st, false, a));
    r = launch_merge<T>(pp, s, ws, va32, nullptr, st, false, ml);
    if (r != AA_OK) return r;
    return backward_gradients<T>(p, q, k, v, agents, dout, dq, dk, dv, dagents, a32, va32, ml,
                                 dva, da, dqa, ej, st);
  };
  rc = run();
  cudaError_t e = cudaFreeAsync(ws, st);
  if (rc == AA_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  return rc;
}

// Fixed scratch of agent_attn_stage_aggregate_static: a file-scope device
// array, so that entry point needs no allocation at all.  Its device address
// is looked up once per device (with that device current) and cached.
static __device__ __align__(256) unsigned char g_static_scratch[AA_STATIC_SCRATCH_BYTES];
std::atomic<void*> g_static_scratch_addr[kMaxDevices];

int static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= 0 && dev < kMaxDevices) {
    void* p = g_static_scratch_addr[dev].load(std::memory_order_acquire);
    if (p != nullptr) {
      *out = p;
      return AA_OK;
    }
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
  if (dev >= 0 && dev < kMaxDevices) g_static_scratch_addr[dev].store(p, std::memory_order_release);
  *out = p;
  return AA_OK;
}

// One FMA-pipe exponential and one exp2f per element (agent_attn_selftest_exp2).
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y_fma,
                                     float* __restrict__ y_ref, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float a = x[i], b = x[i];
  tc::exp2_fma2(a, b);
  y_fma[i] = a;
  y_ref[i] = exp2f(x[i]);
}

}  // namespace
}  // namespace aa

using namespace aa;

extern "C" {

int agent_attn_forward(const void* q, const void* k, const void* v, const void* agents_or_null,
                       void* out, int B, int H, int N, int d, int grid_h, int grid_w, int pool_h,
                       int pool_w, float scale, int dtype, void* stream) {
  return pooled_forward(q, k, v, agents_or_null, out, B, H, N, d, grid_h, grid_w, pool_h, pool_w,
                        scale, dtype, nullptr, 0, false, stream);
}

int agent_attn_forward_ws(const void* q, const void* k, const void* v, const void* agents_or_null,
                          void* out, int B, int H, int N, int d, int grid_h, int grid_w,
                          int pool_h, int pool_w, float scale, int dtype, void* workspace,
                          size_t ws_bytes, void* stream) {
  return pooled_forward(q, k, v, agents_or_null, out, B, H, N, d, grid_h, grid_w, pool_h, pool_w,
                        scale, dtype, workspace, ws_bytes, true, stream);
}

int agent_attn_forward_agents(const void* q, const void* k, const void* v, const void* agents,
                              int n_agents, long long agents_batch_stride, void* out, int B,
                              int H, int N, int d, float scale, int dtype, void* stream) {
  int rc = validate_common(B, H, N, d, n_agents, scale, dtype);
  if (rc != AA_OK) return rc;
  rc = check_tensor_ptrs(q, k, v, out);
  if (rc != AA_OK) return rc;
  if (!agents) return AA_ERR_NULL;
  if (!aligned16(agents)) return AA_ERR_ALIGN;
  if (agents_batch_stride < 0 || (agents_batch_stride % 8) != 0) return AA_ERR_ALIGN;
  Problem p{B, H, N, d, n_agents, 0, 0, 0, 0, scale, dtype};
  AgentsRef learn{agents, agents_batch_stride, (long long)n_agents * d};
  return forward_impl(p, q, k, v, &learn, out, nullptr, 0, false,
                      static_cast<cudaStream_t>(stream));
}

size_t agent_attn_workspace_bytes(int B, int H, int N, int d, int n_agents, int dtype) {
  if (validate_common(B, H, N, d, n_agents, 1.0f, dtype) != AA_OK) return 0;
  int sms = 0;
  if (device_sm_count(&sms) != AA_OK) return 0;
  Problem p{B, H, N, d, n_agents, 0, 0, 0, 0, 1.0f, dtype};
  Scratch s;
  plan_scratch(p, sms, &s);
  return s.total;
}

int agent_attn_forward_host(const void* q_host, const void* k_host, const void* v_host,
                            const void* agents_host_or_null, void* out_host, int B, int H, int N,
                            int d, int grid_h, int grid_w, int pool_h, int pool_w, float scale,
                            int dtype, void* stream) {
  int rc = validate_grid(N, grid_h, grid_w, pool_h, pool_w);
  if (rc != AA_OK) return rc;
  const int kk = pool_h * pool_w;
  rc = validate_common(B, H, N, d, kk, scale, dtype);
  if (rc != AA_OK) return rc;
  if (!q_host || !k_host || !v_host || !out_host) return AA_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t st2 = nullptr;
  rc = side_stream(&st2);
  if (rc != AA_OK) return rc;
  const size_t eb = dtype == AA_FP32 ? 4 : 2;
  const size_t tbytes = round256((size_t)B * H * N * d * eb);
  const size_t abytes = agents_host_or_null ? round256((size_t)H * kk * d * eb) : 0;
  char* dev = nullptr;
  rc = scratch_alloc(reinterpret_cast<void**>(&dev), 4 * tbytes + abytes, st);
  if (rc != AA_OK) return rc;
  char *dq = dev, *dk = dev + tbytes, *dv = dev + 2 * tbytes, *dout = dev + 3 * tbytes;
  char* da = agents_host_or_null ? dev + 4 * tbytes : nullptr;
  // The slices are independent: cut them into chunks (whole batches when the
  // agents are per head) and pipeline chunk c's upload, forward pass and
  // download on one of two streams, so uploads overlap the previous chunk's
  // compute and download (the link is full duplex).
  const long long units = agents_host_or_null ? B : (long long)B * H;
  const long long per_unit = agents_host_or_null ? (long long)H : 1;   // slices per unit
  const long long n_chunks = units < 8 ? units : 8;
  const size_t slice_bytes = (size_t)N * d * eb;
  cudaEvent_t ev_alloc = nullptr, ev_done = nullptr;
  cudaError_t e = cudaEventCreateWithFlags(&ev_alloc, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming);
  if (e == cudaSuccess && da)
    e = cudaMemcpyAsync(da, agents_host_or_null, (size_t)H * kk * d * eb, cudaMemcpyHostToDevice,
                        st);
  if (e == cudaSuccess) e = cudaEventRecord(ev_alloc, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st2, ev_alloc, 0);
  if (e != cudaSuccess) rc = cuda_fail(e, "host pipeline setup");
  for (long long c = 0; c < n_chunks && rc == AA_OK; ++c) {
    const long long u0 = c * units / n_chunks, u1 = (c + 1) * units / n_chunks;
    const size_t off = (size_t)(u0 * per_unit) * slice_bytes;
    const size_t len = (size_t)((u1 - u0) * per_unit) * slice_bytes;
    cudaStream_t cs = (c & 1) ? st2 : st;
    e = cudaMemcpyAsync(dq + off, static_cast<const char*>(q_host) + off, len,
                        cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dk + off, static_cast<const char*>(k_host) + off, len,
                          cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dv + off, static_cast<const char*>(v_host) + off, len,
                          cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) {
      rc = cuda_fail(e, "cudaMemcpyAsync(host to device)");
      break;
    }
    const int cb = agents_host_or_null ? (int)(u1 - u0) : (int)(u1 - u0);
    const int ch = agents_host_or_null ? H : 1;
    rc = pooled_forward(dq + off, dk + off, dv + off, da, dout + off, cb, ch, N, d, grid_h,
                        grid_w, pool_h, pool_w, scale, dtype, nullptr, 0, false, cs);
    if (rc != AA_OK) break;
    e = cudaMemcpyAsync(static_cast<char*>(out_host) + off, dout + off, len,
                        cudaMemcpyDeviceToHost, cs);
    if (e != cudaSuccess) rc = cuda_fail(e, "cudaMemcpyAsync(device to host)");
  }
  // the side stream's work ends before the buffers go back to the pool
  cudaError_t e1 = cudaEventRecord(ev_done, st2);
  if (e1 == cudaSuccess) e1 = cudaStreamWaitEvent(st, ev_done, 0);
  if (rc == AA_OK && e1 != cudaSuccess) rc = cuda_fail(e1, "host pipeline join");
  cudaError_t e2 = cudaFreeAsync(dev, st);
  if (rc == AA_OK && e2 != cudaSuccess) rc = cuda_fail(e2, "cudaFreeAsync");
  cudaError_t e3 = cudaStreamSynchronize(st);
  if (rc == AA_OK && e3 != cudaSuccess) rc = cuda_fail(e3, "cudaStreamSynchronize");
  if (ev_alloc) cudaEventDestroy(ev_alloc);
  if (ev_done) cudaEventDestroy(ev_done);
  return rc;
}

int agent_attn_stage_pool(const void* q, float* agents_f32, void* agents_lowp, int B, int H, int N,
                          int d, int grid_h, int grid_w, int pool_h, int pool_w, int dtype,
                          void* stream) {
  int rc = validate_grid(N, grid_h, grid_w, pool_h, pool_w);
  if (rc != AA_OK) return rc;
  rc = validate_common(B, H, N, d, pool_h * pool_w, 1.0f, dtype);
  if (rc != AA_OK) return rc;
  if (!q) return AA_ERR_NULL;
  if (dtype == AA_FP32) agents_lowp = nullptr;
  if (!agents_f32 && !agents_lowp) return AA_ERR_NULL;
  if (!aligned16(q) || !aligned16(agents_f32) || !aligned16(agents_lowp)) return AA_ERR_ALIGN;
  Problem p{B, H, N, d, pool_h * pool_w, grid_h, grid_w, pool_h, pool_w, 1.0f, dtype};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == AA_FP32) return launch_pool<float>(p, q, agents_f32, nullptr, st);
  return launch_pool<__nv_bfloat16>(p, q, agents_f32, static_cast<__nv_bfloat16*>(agents_lowp),
                                    st);
}

int agent_attn_stage_aggregate(const void* agents, long long agents_batch_stride, const void* k,
                               const void* v, float* va_f32, void* va_lowp, int B, int H, int N,
                               int d, int n_agents, float scale, int dtype, void* stream) {
  int rc = validate_common(B, H, N, d, n_agents, scale, dtype);
  if (rc != AA_OK) return rc;
  if (!agents || !k || !v) return AA_ERR_NULL;
  if (dtype == AA_FP32) va_lowp = nullptr;
  if (!va_f32 && !va_lowp) return AA_ERR_NULL;
  if (!aligned16(agents) || !aligned16(k) || !aligned16(v) || !aligned16(va_f32) ||
      !aligned16(va_lowp))
    return AA_ERR_ALIGN;
  if (agents_batch_stride < 0 || (agents_batch_stride % 8) != 0) return AA_ERR_ALIGN;
  int sms = 0;
  rc = device_sm_count(&sms);
  if (rc != AA_OK) return rc;
  Problem p{B, H, N, d, n_agents, 0, 0, 0, 0, scale, dtype};
  Scratch s;
  plan_scratch(p, sms, &s);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = nullptr;
  rc = scratch_alloc(reinterpret_cast<void**>(&ws), s.total, st);
  if (rc != AA_OK) return rc;
  AgentsRef ag{agents, agents_batch_stride, (long long)n_agents * d};
  rc = (dtype == AA_FP32)
           ? run_aggregate<float>(p, s, ag, k, v, ws, va_f32, nullptr, st)
           : run_aggregate<__nv_bfloat16>(p, s, ag, k, v, ws, va_f32,
                                          static_cast<__nv_bfloat16*>(va_lowp), st);
  cudaError_t e = cudaFreeAsync(ws, st);
  if (rc == AA_OK && e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
  return rc;
}

int agent_attn_stage_aggregate_static(const void* agents, long long agents_batch_stride,
                                      const void* k, const void* v, float* va_f32, void* va_lowp,
                                      int B, int H, int N, int d, int n_agents, float scale,
                                      int dtype, void* stream) {
  int rc = validate_common(B, H, N, d, n_agents, scale, dtype);
  if (rc != AA_OK) return rc;
  if (!agents || !k || !v) return AA_ERR_NULL;
  if (dtype == AA_FP32) va_lowp = nullptr;
  if (!va_f32 && !va_lowp) return AA_ERR_NULL;
  if (!aligned16(agents) || !aligned16(k) || !aligned16(v) || !aligned16(va_f32) ||
      !aligned16(va_lowp))
    return AA_ERR_ALIGN;
  if (agents_batch_stride < 0 || (agents_batch_stride % 8) != 0) return AA_ERR_ALIGN;
  int sms = 0;
  rc = device_sm_count(&sms);
  if (rc != AA_OK) return rc;
  Problem p{B, H, N, d, n_agents, 0, 0, 0, 0, scale, dtype};
  Scratch s;
  plan_scratch(p, sms, &s);
  // The aggregation touches only the partial-state regions [pu_off, total) of
  // the scratch layout: a copy of the plan with those regions moved to offset
  // 0 addresses the fixed array from its start (the agent and V_A regions,
  // which the aggregation does not use, are left empty).
  const size_t need = s.total - s.pu_off;
  if (need > (size_t)AA_STATIC_SCRATCH_BYTES) return AA_ERR_WORKSPACE;
  Scratch r = s;
  r.a_off = r.va_off = r.b1d_off = r.b2d_off = r.b2t_off = 0;
  r.pml_off = s.pml_off - s.pu_off;
  r.pu_off = 0;
  r.total = need;
  void* base = nullptr;
  rc = static_scratch_address(&base);
  if (rc != AA_OK) return rc;
  char* ws = static_cast<char*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  AgentsRef ag{agents, agents_batch_stride, (long long)n_agents * d};
  return (dtype == AA_FP32)
             ? run_aggregate<float>(p, r, ag, k, v, ws, va_f32, nullptr, st)
             : run_aggregate<__nv_bfloat16>(p, r, ag, k, v, ws, va_f32,
                                            static_cast<__nv_bfloat16*>(va_lowp), st);
}

int agent_attn_stage_broadcast(const void* q, const void* agents, long long agents_batch_stride,
                               const void* va, void* out, int B, int H, int N, int d,
                               int n_agents, float scale, int dtype, void* stream) {
  int rc = validate_common(B, H, N, d, n_agents, scale, dtype);
  if (rc != AA_OK) return rc;
  if (!q || !agents || !va || !out) return AA_ERR_NULL;
  if (!aligned16(q) || !aligned16(agents) || !aligned16(va) || !aligned16(out))
    return AA_ERR_ALIGN;
  if (agents_batch_stride < 0 || (agents_batch_stride % 8) != 0) return AA_ERR_ALIGN;
  Problem p{B, H, N, d, n_agents, 0, 0, 0, 0, scale, dtype};
  AgentsRef ag{agents, agents_batch_stride, (long long)n_agents * d};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (dtype == AA_FP32) ? run_broadcast<float>(p, q, ag, va, out, st)
                            : run_broadcast<__nv_bfloat16>(p, q, ag, va, out, st);
}

const char* agent_attn_status_string(int status) {
  switch (status) {
    case AA_OK: return "AA_OK: success";
    case AA_ERR_NULL: return "AA_ERR_NULL: a required pointer is NULL";
    case AA_ERR_SHAPE: return "AA_ERR_SHAPE: inconsistent sizes (N vs grid, pool vs grid, B/H/N)";
    case AA_ERR_UNSUPPORTED: return "AA_ERR_UNSUPPORTED: dtype, head dim d or agent count k not supported";
    case AA_ERR_ALIGN: return "AA_ERR_ALIGN: pointer or stride not aligned as required";
    case AA_ERR_WORKSPACE: return "AA_ERR_WORKSPACE: caller workspace too small";
    case AA_ERR_CUDA: return g_cuda_err;
    case AA_ERR_VALUE: return "AA_ERR_VALUE: scale must be finite and > 0";
    case AA_ERR_TIMEOUT:
      return "AA_ERR_TIMEOUT: a kernel's bounded wait expired (pipeline stalled); results invalid";
    default: return "unknown agent_attn status";
  }
}

const char* agent_attn_version(void) { return "0.1.0"; }

int agent_attn_selftest_exp2(const float* x, float* y_fma, float* y_ref, int n, void* stream) {
  if (n < 0) return AA_ERR_SHAPE;
  if (n == 0) return AA_OK;
  if (!x || !y_fma || !y_ref) return AA_ERR_NULL;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y_fma) |
                        reinterpret_cast<uintptr_t>(y_ref);
  if (mis & 3u) return AA_ERR_ALIGN;
  selftest_exp2_kernel<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y_fma, y_ref, n);
  AA_CUDA(cudaGetLastError());
  return AA_OK;
}

int agent_attn_dwc(const void* v, const float* w, const float* bias_or_null, void* out, int B,
                   int H, int grid_h, int grid_w, int d, int dtype, int accumulate, void* stream) {
  int rc = validate_dwc(v, w, out, B, H, grid_h, grid_w, d, dtype);
  if (rc != AA_OK) return rc;
  if (bias_or_null && (reinterpret_cast<uintptr_t>(bias_or_null) & 3u)) return AA_ERR_ALIGN;
  return dwc_impl(v, w, bias_or_null, out, B, H, grid_h, grid_w, d, dtype, accumulate ? 1 : 0,
                  static_cast<cudaStream_t>(stream), false);
}

int agent_attn_forward_dwc(const void* q, const void* k, const void* v, const void* agents_or_null,
                           const float* dwc_w, const float* dwc_bias_or_null, void* out, int B,
                           int H, int N, int d, int grid_h, int grid_w, int pool_h, int pool_w,
                           float scale, int dtype, void* stream) {
  int rc = validate_grid(N, grid_h, grid_w, pool_h, pool_w);
  if (rc != AA_OK) return rc;
  rc = validate_dwc(v, dwc_w, out, B, H, grid_h, grid_w, d, dtype);
  if (rc != AA_OK) return rc;
  if (dwc_bias_or_null && (reinterpret_cast<uintptr_t>(dwc_bias_or_null) & 3u)) return AA_ERR_ALIGN;
  rc = pooled_forward(q, k, v, agents_or_null, out, B, H, N, d, grid_h, grid_w, pool_h, pool_w,
                      scale, dtype, nullptr, 0, false, stream);
  if (rc != AA_OK) return rc;
  return dwc_impl(v, dwc_w, dwc_bias_or_null, out, B, H, grid_h, grid_w, d, dtype, 1,
                  static_cast<cudaStream_t>(stream), true);
}

int agent_attn_forward_bias(const void* q, const void* k, const void* v, const void* agents_or_null,
                            const float* b1_row, const float* b1_col, const float* b1_block,
                            const float* b2_row, const float* b2_col, const float* b2_block,
                            void* out, int B, int H, int N, int d, int grid_h, int grid_w,
                            int pool_h, int pool_w, float scale, int dtype, void* stream) {
  int rc = validate_grid(N, grid_h, grid_w, pool_h, pool_w);
  if (rc != AA_OK) return rc;
  const int kk = pool_h * pool_w;
  rc = validate_common(B, H, N, d, kk, scale, dtype);
  if (rc != AA_OK) return rc;
  rc = check_tensor_ptrs(q, k, v, out);
  if (rc != AA_OK) return rc;
  if (agents_or_null && !aligned16(agents_or_null)) return AA_ERR_ALIGN;
  const float* parts[6] = {b1_row, b1_col, b1_block, b2_row, b2_col, b2_block};
  for (const float* b : parts)
    if (b && (reinterpret_cast<uintptr_t>(b) & 3u)) return AA_ERR_ALIGN;
  AgentBiasRef bias1{b1_row, b1_col, b1_block}, bias2{b2_row, b2_col, b2_block};
  Problem p{B, H, N, d, kk, grid_h, grid_w, pool_h, pool_w, scale, dtype};
  p.b1 = &bias1;
  p.b2 = &bias2;
  AgentsRef learn{agents_or_null, 0, (long long)kk * d};
  return forward_impl(p, q, k, v, agents_or_null ? &learn : nullptr, out, nullptr, 0, false,
                      static_cast<cudaStream_t>(stream));
}

int agent_attn_backward(const void* q, const void* k, const void* v, const void* agents_or_null,
                        const void* dout, void* dq, void* dk, void* dv, float* dagents_or_null,
                        int B, int H, int N, int d, int grid_h, int grid_w, int pool_h, int pool_w,
                        float scale, int dtype, void* stream) {
  int rc = validate_grid(N, grid_h, grid_w, pool_h, pool_w);
  if (rc != AA_OK) return rc;
  const int kk = pool_h * pool_w;
  rc = validate_common(B, H, N, d, kk, scale, dtype);
  if (rc != AA_OK) return rc;
  rc = check_tensor_ptrs(q, k, v, dout);
  if (rc != AA_OK) return rc;
  if (!dq || !dk || !dv) return AA_ERR_NULL;
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return AA_ERR_ALIGN;
  if (agents_or_null && !aligned16(agents_or_null)) return AA_ERR_ALIGN;
  if (dagents_or_null && (reinterpret_cast<uintptr_t>(dagents_or_null) & 3u)) return AA_ERR_ALIGN;
  if ((long long)B * H > 65535) return AA_ERR_SHAPE;
  Problem p{B, H, N, d, kk, grid_h, grid_w, pool_h, pool_w, scale, dtype};
  p.force_simt = true;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == AA_FP32
             ? backward_impl<float>(p, q, k, v, agents_or_null, dout, dq, dk, dv, dagents_or_null,
                                    st)
             : backward_impl<__nv_bfloat16>(p, q, k, v, agents_or_null, dout, dq, dk, dv,
                                            dagents_or_null, st);
}

int agent_attn_check_device_error(void) {
  unsigned int word = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&word, tc::g_watchdog, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(watchdog)");
  if (word == 0) return AA_OK;
  e = cudaMemcpyToSymbol(tc::g_watchdog, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(watchdog)");
  return AA_ERR_TIMEOUT;
}

}  // extern "C"
