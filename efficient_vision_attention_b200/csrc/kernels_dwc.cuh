// Depth-wise 3x3 convolution of V over the token grid, added to the attention
// output: the DWC term of the full Agent Attention module (the arXiv
// 2312.08874v3 summary, §4 "Module Enhancements": a depth-wise convolution
// term of cost k^2 N C with k = 3).
//
// Two kernels.  dwc_stream_kernel (below; used whenever B*H fits the grid's y
// extent) streams V rows through a shared-memory ring with bulk copies and
// convolves from there.  dwc_kernel reads the taps through L1/L2 and streams
// any number of slices:
// each thread owns a run of kDwcSpan neighbouring tokens of one grid row and
// one 8-channel group of a (batch, head) slice: it reads the 3 x (kDwcSpan+2)
// neighbouring 8-channel groups of V once (zero outside the grid), applies the
// head's per-channel 3x3 kernels (staged in shared memory as [tap][channel],
// each weight vector read once for the whole run), adds the bias and, when
// accumulating, the value already in `out`, and writes the run.  Consecutive
// threads cover consecutive channel groups of consecutive runs, so every tap
// row is a coalesced read and blocks share rows through L1/L2.  HBM-bound:
// V read once, out read (when accumulating) and written once.
#pragma once

#include "common.cuh"
#include "tc_primitives.cuh"

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

// Tokens per thread along x: neighbouring outputs share 2 of their 3 tap
// columns and every weight vector.
constexpr int kDwcSpan = 2;

// v, out: [BH][grid_h*grid_w][d] of T; w: [H][d][3][3] fp32; bias: [H][d] fp32
// or null.  Thread = (grid row y, run of kDwcSpan tokens along x, 8-channel
// group); grid: (ceil(items / kDwcThreads), min(BH, 65535)) with
// items = grid_h * ceil(grid_w / kDwcSpan) * d/8 < 2^31.  With programmatic
// dependent launch the convolution is computed before waiting for the
// previous kernel of the stream (which writes `out`, not V).
template <typename T>
__global__ void __launch_bounds__(kDwcThreads)
    dwc_kernel(const T* __restrict__ v, const float* __restrict__ w,
               const float* __restrict__ bias, T* __restrict__ out, int H, int grid_h,
               int grid_w, int d, long long BH, int accumulate) {
  extern __shared__ float s_w[];   // [9][d] kernel taps, then [d] bias
  pdl_trigger();
  const unsigned nch = (unsigned)d / 8u;
  const unsigned xruns = ((unsigned)grid_w + kDwcSpan - 1) / kDwcSpan;
  const unsigned N = (unsigned)grid_h * (unsigned)grid_w;
  const unsigned items = (unsigned)grid_h * xruns * nch;
  const unsigned item = blockIdx.x * blockDim.x + threadIdx.x;
  const bool mine = item < items;
  const unsigned ch = mine ? item % nch : 0u;
  const unsigned run = mine ? item / nch : 0u;
  const int y = (int)(run / xruns);
  const int x0 = (int)(run - (unsigned)y * xruns) * kDwcSpan;
  for (long long bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const int h = (int)(bh % H);
    __syncthreads();   // the previous slice's weights are no longer read
    for (int i = threadIdx.x; i < 9 * d; i += blockDim.x) {
      const int tap = i / d, c = i - tap * d;
      s_w[i] = w[((long long)h * d + c) * 9 + tap];
    }
    for (int i = threadIdx.x; i < d; i += blockDim.x) s_w[9 * d + i] = bias ? bias[h * d + i] : 0.f;
    __syncthreads();
    float acc[kDwcSpan][8];
    const T* vs = v + bh * (long long)N * d + ch * 8;
    if (mine) {
#pragma unroll
      for (int t = 0; t < kDwcSpan; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[t][e] = s_w[9 * d + ch * 8 + e];
#pragma unroll
      for (int ty = 0; ty < 3; ++ty) {
        const int yy = y + ty - 1;
        if (yy < 0 || yy >= grid_h) continue;
        // the kDwcSpan + 2 tap columns x0-1 .. x0+kDwcSpan of row yy, kept as
        // raw 16-byte rows and widened at each use (fewer live registers)
        uint4 raw[kDwcSpan + 2];
        const T* cp[kDwcSpan + 2];
        bool cin[kDwcSpan + 2];
#pragma unroll
        for (int c = 0; c < kDwcSpan + 2; ++c) {
          const int xx = x0 + c - 1;
          cin[c] = xx >= 0 && xx < grid_w;
          cp[c] = vs + (size_t)((unsigned)yy * grid_w + (cin[c] ? xx : 0)) * d;
          raw[c] = cin[c] ? load16(cp[c]) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int tx = 0; tx < 3; ++tx) {
          float wt[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) wt[e] = s_w[(ty * 3 + tx) * d + ch * 8 + e];
#pragma unroll
          for (int t = 0; t < kDwcSpan; ++t) {
            if (!cin[t + tx]) continue;
            float cv[8];
            unpack8(raw[t + tx], cp[t + tx], cv);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[t][e] = fmaf(wt[e], cv[e], acc[t][e]);
          }
        }
      }
    }
    pdl_wait();   // `out` may be written by the previous kernel of the stream
    if (mine) {
#pragma unroll
      for (int t = 0; t < kDwcSpan; ++t) {
        if (x0 + t >= grid_w) continue;
        T* o = out + (bh * (long long)N + (long long)y * grid_w + x0 + t) * d + ch * 8;
        if (accumulate) {
          float prev[8];
          load8(o, prev);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[t][e] += prev[e];
        }
        store8(o, acc[t]);
      }
    }
  }
}

// ------------------------------------------------ streaming variant
// CTA = (slice, chunk of token columns, band of output rows); thread = (run
// of kDwcTok neighbouring tokens, 8-channel group), the same item on every
// row, so the block is one row of items.  The CTA walks its band top to
// bottom.  V rows live in a ring of kDwcRing shared-memory slots (each the
// chunk's columns plus a one-column halo on each side); thread 0 keeps the
// ring filled two rows ahead of the computation with one bulk copy per row,
// each onto its slot's mbarrier.  Output row y reads V rows y-1, y, y+1 from
// the ring: each of the kDwcTok+2 tap columns of a row is widened once and
// feeds up to three outputs on the paired FP32 datapath.  When accumulating,
// a thread loads its part of out row y+1 into registers while it computes
// row y, and starts row y+1's sums from it (with the bias).  After each row
// the CTA votes at one barrier, which also frees the slot of V row y-2 for
// the refill.  Every V row is read from HBM once per CTA (band edges once
// more, from L2).
constexpr int kDwcTok = 4;
constexpr int kDwcRing = 5;      // V rows resident: y-1, y, y+1 and two in flight
constexpr int kDwcMaxThreads = 512;
constexpr int kDwcSmemBudget = 100 * 1024;
// Row y+1 is issued at the latest after the vote of step y+3-kDwcRing, so
// strictly before step y waits for it.
static_assert(kDwcRing >= 4, "ring too short for the refill schedule");

struct DwcStreamPlan {
  int cols;             // token columns per chunk
  int n_xc;             // column chunks
  int threads;          // one row of items, rounded up to whole warps
  int vslot;            // slot size in elements (a multiple of 128 bytes)
  size_t smem;
  bool ok;
};

// Column chunking and block shape; the row bands follow from the occupancy
// (dwc_stream_bands).
inline DwcStreamPlan dwc_stream_plan(int grid_w, int d, int elem) {
  DwcStreamPlan pl{};
  const size_t row_tok = (size_t)d * elem;
  auto round128 = [](size_t b) { return (b + 127) & ~(size_t)127; };
  auto bytes = [&](int c) {
    return 128 + kDwcRing * round128((size_t)(c + 2) * row_tok) + (size_t)10 * d * sizeof(float) +
           kDwcRing * sizeof(uint64_t);
  };
  auto items = [&](int c) { return ((c + kDwcTok - 1) / kDwcTok) * (d / 8); };
  int cols = grid_w;
  while (cols > 1 && (bytes(cols) > (size_t)kDwcSmemBudget || items(cols) > kDwcMaxThreads))
    cols = (cols + 1) / 2;
  if (bytes(cols) > (size_t)kDwcSmemBudget || items(cols) > kDwcMaxThreads) return pl;
  pl.cols = cols;
  pl.n_xc = (grid_w + cols - 1) / cols;
  pl.threads = (items(cols) + 31) & ~31;
  pl.vslot = (int)(round128((size_t)(cols + 2) * row_tok) / elem);
  pl.smem = bytes(cols);
  pl.ok = true;
  return pl;
}

// Rows per band so that all CTAs are resident at once when the slices allow
// (at least kDwcMinBand rows, so the halo rows stay a minor share).
constexpr int kDwcMinBand = 4;
inline int dwc_stream_band(int grid_h, long long units, long long resident) {
  const long long per_unit = units >= resident ? 1 : resident / units;
  int band = (int)((grid_h + per_unit - 1) / per_unit);
  if (band < kDwcMinBand) band = kDwcMinBand;
  return band < grid_h ? band : grid_h;
}

// Raw 8-channel group of one token (16 bytes for bf16, 32 for fp32).
template <typename T> struct DwcRaw;
template <> struct DwcRaw<__nv_bfloat16> {
  uint4 a;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    a = *reinterpret_cast<const uint4*>(p);
  }
  __device__ __forceinline__ void zero() { a = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void widen(float2 (&f)[4]) const {
    const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      f[i] = make_float2(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
  }
};
template <> struct DwcRaw<float> {
  uint4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = *reinterpret_cast<const uint4*>(p);
    b = *reinterpret_cast<const uint4*>(p + 4);
  }
  __device__ __forceinline__ void zero() { a = b = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void widen(float2 (&f)[4]) const {
    f[0] = make_float2(__uint_as_float(a.x), __uint_as_float(a.y));
    f[1] = make_float2(__uint_as_float(a.z), __uint_as_float(a.w));
    f[2] = make_float2(__uint_as_float(b.x), __uint_as_float(b.y));
    f[3] = make_float2(__uint_as_float(b.z), __uint_as_float(b.w));
  }
};

// grid: (n_bands * n_xc, BH <= 65535); block: plan.threads; dynamic shared
// memory: plan.smem.
template <typename T>
__global__ void __launch_bounds__(kDwcMaxThreads)
    dwc_stream_kernel(const T* __restrict__ v, const float* __restrict__ w,
                      const float* __restrict__ bias, T* __restrict__ out, int H, int grid_h,
                      int grid_w, int d, int cols, int band, int vslot, int accumulate) {
  extern __shared__ uint8_t dwc_smem[];
  pdl_trigger();
  // 128-byte aligned by pointer arithmetic on the shared array, so the
  // compiler keeps the shared address space for every access through it
  uint8_t* base = dwc_smem + ((128u - (tc::smem_u32(dwc_smem) & 127u)) & 127u);
  T* vring = reinterpret_cast<T*>(base);                                   // [kDwcRing][vslot]
  float* s_w = reinterpret_cast<float*>(vring + (size_t)kDwcRing * vslot);  // [9][d], [d]
  uint64_t* vbar = reinterpret_cast<uint64_t*>(s_w + 10 * d);
  const int n_xc = (grid_w + cols - 1) / cols;
  const int bi = blockIdx.x / n_xc, xc = blockIdx.x - bi * n_xc;
  const int ya = bi * band, yb = min(ya + band, grid_h);
  const int xs = xc * cols, xw = min(cols, grid_w - xs);
  const long long bh = blockIdx.y;
  const int h = (int)(bh % H);
  const long long N = (long long)grid_h * grid_w;
  // V rows ya-1 .. yb (inside the grid) over grid columns [sx0, sx1); slot
  // column j holds grid column xs-1+j.  V row r uses slot (r-ya+1) % kDwcRing.
  const int vhi = min(yb, grid_h - 1);
  const int sx0 = max(xs - 1, 0), sx1 = min(xs + xw + 1, grid_w);
  const uint32_t vbytes = (uint32_t)((size_t)(sx1 - sx0) * d * sizeof(T));
  auto vslot_of = [&](int r) { return (r - ya + 1) % kDwcRing; };
  auto vpar_of = [&](int r) { return (uint32_t)(((r - ya + 1) / kDwcRing) & 1); };
  auto issue_v = [&](int r) {   // thread 0 only
    if (r > vhi) return;
    uint64_t* bar = vbar + vslot_of(r);
    if (r < 0) {   // the row above the grid: complete the slot's phase empty
      tc::mbar_arrive(bar);
      return;
    }
    T* dst = vring + (size_t)vslot_of(r) * vslot + (size_t)(sx0 - (xs - 1)) * d;
    const T* src = v + (bh * N + (long long)r * grid_w + sx0) * d;
    tc::mbar_expect_tx(bar, vbytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];" ::"r"(tc::smem_u32(dst)),
        "l"(src), "r"(vbytes), "r"(tc::smem_u32(bar))
        : "memory");
  };
  auto wait_row = [&](int r) {   // bounded; false after the limit
    uint64_t* bar = vbar + vslot_of(r);
    const uint32_t par = vpar_of(r);
    if (tc::mbar_try_wait(bar, par)) return true;
    const uint64_t t0 = tc::globaltimer();
    while (!tc::mbar_try_wait(bar, par)) {
      if (tc::globaltimer() - t0 > tc::kWaitLimitNs) {
        atomicOr(&tc::g_watchdog, 1u);
        return false;
      }
    }
    return true;
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDwcRing; ++i) tc::mbar_init(vbar + i, 1);
    tc::mbar_fence_init();
    for (int r = ya - 1; r < ya - 1 + kDwcRing; ++r) issue_v(r);
  }
  for (int i = threadIdx.x; i < 9 * d; i += blockDim.x) {
    const int tap = i / d, c = i - tap * d;
    s_w[i] = w[((long long)h * d + c) * 9 + tap];
  }
  for (int i = threadIdx.x; i < d; i += blockDim.x) s_w[9 * d + i] = bias ? bias[h * d + i] : 0.f;

  const int nch = d >> 3;
  const int items = ((xw + kDwcTok - 1) / kDwcTok) * nch;
  const bool mine = (int)threadIdx.x < items;
  const int ch = (int)threadIdx.x % nch;
  const int x0 = ((int)threadIdx.x / nch) * kDwcTok;   // chunk-relative first token
  T* orow = out + (bh * N + xs + x0) * d + ch * 8;      // + y * grid_w * d: token x0 of row y
  DwcRaw<T> pre[kDwcTok];
  auto load_prev = [&](int y) {
#pragma unroll
    for (int t = 0; t < kDwcTok; ++t) {
      if (x0 + t < xw) pre[t].load(orow + ((long long)y * grid_w + t) * d);
      else pre[t].zero();
    }
  };
  pdl_wait();   // `out` may be written by the previous kernel of the stream
  if (mine && accumulate) load_prev(ya);
  __syncthreads();   // barriers initialised, weights staged

  // slot columns x0 .. x0+kDwcTok+1 = grid columns xs+x0-1 .. xs+x0+kDwcTok;
  // bit c of cmask: column x0+c is inside the grid and staged (else it adds 0)
  unsigned cmask = 0;
#pragma unroll
  for (int c = 0; c < kDwcTok + 2; ++c) {
    const int j = x0 + c, gx = xs - 1 + j;
    if (gx >= 0 && gx < grid_w && j <= xw + 1) cmask |= 1u << c;
  }
  const T* vcol = vring + (size_t)x0 * d + ch * 8;               // + slot * vslot + c * d
  const float4* w4 = reinterpret_cast<const float4*>(s_w + ch * 8);  // + tap * d/4
  const int dq = d >> 2;

  bool ok = true;
  int y = ya;
  int s0 = 0;   // ring slot of V row y-1 (slots of rows y, y+1 follow cyclically)
  for (; y < yb; ++y, s0 = (s0 + 1 == kDwcRing) ? 0 : s0 + 1) {
    for (int r = max(y - 1, 0); r <= min(y + 1, grid_h - 1); ++r) ok = ok && wait_row(r);
    // one vote per row: every thread has finished row y-1 (the slot of V
    // row y-2 is free) and sees row y's loads complete
    if (__syncthreads_or(!ok)) break;
    if (threadIdx.x == 0 && y > ya) issue_v(y - 2 + kDwcRing);
    if (!mine) continue;
    float2 acc[kDwcTok][4];
    {
      const float4 b0 = w4[9 * dq], b1 = w4[9 * dq + 1];
      const float2 b2[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w),
                            make_float2(b1.x, b1.y), make_float2(b1.z, b1.w)};
#pragma unroll
      for (int t = 0; t < kDwcTok; ++t) {
        if (accumulate) {
          float2 p[4];
          pre[t].widen(p);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[t][i] = __fadd2_rn(b2[i], p[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[t][i] = b2[i];
        }
      }
    }
    if (accumulate && y + 1 < yb) load_prev(y + 1);   // consumed at the next row
#pragma unroll
    for (int ty = 0; ty < 3; ++ty) {
      const int r = y + ty - 1;
      if (r < 0 || r >= grid_h) continue;
      float2 wv[3][4];
#pragma unroll
      for (int tx = 0; tx < 3; ++tx) {
        const float4 a0 = w4[(ty * 3 + tx) * dq], a1 = w4[(ty * 3 + tx) * dq + 1];
        wv[tx][0] = make_float2(a0.x, a0.y);
        wv[tx][1] = make_float2(a0.z, a0.w);
        wv[tx][2] = make_float2(a1.x, a1.y);
        wv[tx][3] = make_float2(a1.z, a1.w);
      }
      int sl = s0 + ty;
      if (sl >= kDwcRing) sl -= kDwcRing;
      const T* src = vcol + (size_t)sl * vslot;
#pragma unroll
      for (int c = 0; c < kDwcTok + 2; ++c) {
        if (!((cmask >> c) & 1u)) continue;
        DwcRaw<T> raw;
        raw.load(src + c * d);
        float2 cv[4];
        raw.widen(cv);
#pragma unroll
        for (int tx = 0; tx < 3; ++tx) {
          const int t = c - tx;
          if (t < 0 || t >= kDwcTok) continue;
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[t][i] = __ffma2_rn(wv[tx][i], cv[i], acc[t][i]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kDwcTok; ++t) {
      if (x0 + t >= xw) continue;
      const float o8[8] = {acc[t][0].x, acc[t][0].y, acc[t][1].x, acc[t][1].y,
                           acc[t][2].x, acc[t][2].y, acc[t][3].x, acc[t][3].y};
      store8(orow + ((long long)y * grid_w + t) * d, o8);
    }
  }
  if (y < yb && threadIdx.x == 0) {
    // a load outlived the limit: wait (bounded) for every copy still in
    // flight into the ring before this CTA's shared memory is released
    const int vlast = min(max(ya - 2 + kDwcRing, y - 3 + kDwcRing), vhi);
    for (int r = max(vlast - kDwcRing + 1, max(ya - 1, 0)); r <= vlast; ++r) {
      const uint64_t t0 = tc::globaltimer();
      while (!tc::mbar_try_wait(vbar + vslot_of(r), vpar_of(r)) &&
             tc::globaltimer() - t0 < tc::kWaitLimitNs) {
      }
    }
  }
}

}  // namespace aa
