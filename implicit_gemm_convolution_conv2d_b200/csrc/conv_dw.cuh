// conv_dw.cuh -- direct depthwise convolution forward (groups = C = O).
//
// The "Convolutions" tutorial ("Convolution variants worth knowing") lists
// depthwise convolution -- one filter per channel, C_in x K x K weights -- as
// cheap and memory-bound, and its list of alternatives to im2col names direct,
// shape-specialised kernels as the usual choice for it: as an implicit GEMM
// each group would be an N = 1, K = kD*kH*kW product, nothing a tensor core
// can use.  This kernel computes
//   y[n, od, oh, ow, c] = sum_{kd,kh,kw} x[n, od*sd - pd + kd*dd, oh*sh - ph + kh*dh,
//                                          ow*sw - pw + kw*dw, c] * w[c, kd, kh, kw]
// (w read reversed in every spatial dimension when flipped) with fp32 FMAs
// and fp32 accumulation, x and y streamed once through the cache hierarchy.
//
// Work split: a thread owns V consecutive channels (one 16-byte vector of x
// and y) of P consecutive output pixels along W.  A block is CB channel
// vectors x PB pixel groups; consecutive threads take consecutive channel
// vectors of one pixel group, so a warp reads and writes whole runs of a
// pixel's channels.  The block's filters are copied once into shared memory
// as fp32, tap-major, so a thread reads its V weights of a tap as V/4
// conflict-free 16-byte shared loads; in the layout of w (channel-major) the
// same read would touch V scattered elements.
//
// Filter rows: with the filter width, width stride and width dilation known
// at compile time (KW > 0), a thread holds the row's KW weight vectors in
// registers and streams the (P-1)*SW + (KW-1)*DW + 1 input pixels its P
// outputs read from one input row, each loaded once (zero outside the row)
// and applied to every (pixel, kw) pair that reads it.  The generic form
// (KW = 0) issues one load per (pixel, kw) and relies on L1 for the reuse.
#pragma once

#include <cstdint>
#include <cstring>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "conv_simt.cuh"  // to_f32 / from_f32
#include "conv_tc.cuh"    // bounded mbarrier waits, status word
#include "ptx.cuh"

namespace convfwd {

struct DwArgs {
  int N, D, H, W, C;
  int kD, kH, kW;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  int Do, Ho, Wo;
  int wg;        // pixel groups per output row: ceil(Wo / P)
  int flip;      // 1: the filter is read reversed in every spatial dimension
  int cb;        // channel vectors per block (CB)
  int pb;        // pixel groups per block (PB); blockDim.x = CB * PB
  int groups;    // pixel groups in the problem: N * Do * Ho * wg (below 2^31 - 256)
  const void* x;
  const void* w;
  void* y;
};

constexpr int kDwThreads = 256;       // upper bound on CB * PB
constexpr int kDwMaxCB = 32;          // at most one warp of channel vectors per pixel group
constexpr int kDwSmemLimit = 200 * 1024;

template <typename T, int V>
struct DwVec;  // V elements of T as one 16-byte access
template <>
struct DwVec<float, 4> {
  using type = float4;
};
template <>
struct DwVec<__half, 8> {
  using type = uint4;
};
template <>
struct DwVec<__nv_bfloat16, 8> {
  using type = uint4;
};

// Unpacks a 16-byte vector held in registers.  Taken by value: a reference
// to shared memory here would turn into V narrow shared loads.
template <typename T, int V>
__device__ __forceinline__ void dw_unpack(const typename DwVec<T, V>::type raw, float (&f)[V]) {
  const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
  for (int v = 0; v < V; ++v) f[v] = to_f32<T>(e[v]);
}

// Shared-memory filters are fp32 laid out [tap][V/4][CB][4]: for one tap and
// one quad of a thread's V channels, consecutive channel vectors are
// consecutive 16-byte words, so a quarter-warp's reads hit distinct banks.
template <int V>
__device__ __forceinline__ int dw_widx(int tap, int cl, int cb) {
  const int cv = cl / V, e = cl - cv * V;
  return ((tap * (V / 4) + e / 4) * cb + cv) * 4 + (e & 3);
}

// The V weights of one tap for channel vector cv: `p` points at the tap's
// first quad plus cv * 4.
template <int V>
__device__ __forceinline__ void dw_weights(const float* p, int cb, float (&wv)[V]) {
#pragma unroll
  for (int q = 0; q < V / 4; ++q) {
    const float4 t4 = *reinterpret_cast<const float4*>(p + q * cb * 4);
    wv[4 * q] = t4.x;
    wv[4 * q + 1] = t4.y;
    wv[4 * q + 2] = t4.z;
    wv[4 * q + 3] = t4.w;
  }
}

// Two fp32 FMAs as one packed instruction (fma.rn.f32x2, sm_100): each lane
// is an ordinary round-to-nearest fused multiply-add, so the results equal
// two fmaf calls.
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 d, a, b;\n\t"
      "mov.b64 d, {%0, %1};\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %5};\n\t"
      "fma.rn.f32x2 d, a, b, d;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// acc[v] += x[v] * w[v] for v < V, as V/2 packed FMAs.
template <int V>
__device__ __forceinline__ void dw_fma(float (&acc)[V], const float (&x)[V], const float (&w)[V]) {
#pragma unroll
  for (int v = 0; v < V; v += 2) ffma2(acc[v], acc[v + 1], x[v], x[v + 1], w[v], w[v + 1]);
}

// KW, SW, DW: compile-time filter width, width stride and width dilation, or
// all 0 for the runtime form.
template <typename T, int V, int P, int KW, int SW, int DW>
__global__ void __launch_bounds__(kDwThreads, 2) conv_fwd_dw_direct_kernel(const DwArgs a) {
  using Vec = typename DwVec<T, V>::type;
  extern __shared__ __align__(16) float s_w[];  // [taps][V/4][CB][4]
  const int taps = a.kD * a.kH * a.kW;
  const int cbv = a.cb * V;
  const int cbase = blockIdx.y * cbv;  // first channel of the block
  // (no early trigger: several blocks of this kernel share an SM; the next
  // launch starts as they exit)
  ptx::pdl_wait_prev();  // the previous launch's writes are visible from here on

  // Filters of the block's channels, tap-major, mirrored under flip.  Read in
  // w's own order (channel-major) so the global reads are contiguous.
  for (int i = threadIdx.x; i < cbv * taps; i += blockDim.x) {
    const int cl = i / taps;
    const int t = i - cl * taps;
    const int c = cbase + cl;
    s_w[dw_widx<V>(a.flip ? taps - 1 - t : t, cl, a.cb)] =
        c < a.C ? to_f32<T>(static_cast<const T*>(a.w)[static_cast<long long>(c) * taps + t]) : 0.f;
  }
  __syncthreads();

  const int cl = threadIdx.x % a.cb;
  const int grp = static_cast<int>(blockIdx.x) * a.pb + static_cast<int>(threadIdx.x) / a.cb;
  const int c0 = cbase + cl * V;
  if (grp >= a.groups || c0 >= a.C) return;
  int q = grp;  // 32-bit decode: the pixel-group count is below 2^31
  const int g = q % a.wg;
  q /= a.wg;
  const int oh = q % a.Ho;
  q /= a.Ho;
  const int od = q % a.Do;
  const long long n = q / a.Do;
  const int ow0 = g * P;

  const T* __restrict__ x = static_cast<const T*>(a.x);
  T* __restrict__ y = static_cast<T*>(a.y);
  const float* sw_c = s_w + cl * 4;

  float acc[P][V];
#pragma unroll
  for (int p = 0; p < P; ++p)
#pragma unroll
    for (int v = 0; v < V; ++v) acc[p][v] = 0.f;

  for (int kd = 0; kd < a.kD; ++kd) {
    const int id = od * a.sd - a.pd + kd * a.dd;
    if (static_cast<unsigned>(id) >= static_cast<unsigned>(a.D)) continue;
    for (int kh = 0; kh < a.kH; ++kh) {
      const int ih = oh * a.sh - a.ph + kh * a.dh;
      if (static_cast<unsigned>(ih) >= static_cast<unsigned>(a.H)) continue;
      const T* xrow = x + ((n * a.D + id) * a.H + ih) * static_cast<long long>(a.W) * a.C + c0;
      const float* wtap = sw_c + (kd * a.kH + kh) * a.kW * cbv;  // a tap is cbv floats
      if constexpr (KW > 0) {
        // the row's KW weight vectors in registers, then the input columns of
        // the window streamed once each into every (pixel, kw) pair that reads
        // them (the pairing is resolved at compile time)
        constexpr int SPAN = (P - 1) * SW + (KW - 1) * DW + 1;
        float wv[KW][V];
#pragma unroll
        for (int kw = 0; kw < KW; ++kw) dw_weights<V>(wtap + kw * cbv, a.cb, wv[kw]);
        const int iw0 = ow0 * SW - a.pw;
#pragma unroll
        for (int j = 0; j < SPAN; ++j) {
          // columns outside the row load column 0 (in bounds) and read as zero
          const int iw = iw0 + j;
          const bool in = static_cast<unsigned>(iw) < static_cast<unsigned>(a.W);
          const Vec raw = __ldg(reinterpret_cast<const Vec*>(xrow + static_cast<long long>(in ? iw : 0) * a.C));
          float xf[V];
          dw_unpack<T, V>(raw, xf);
#pragma unroll
          for (int v = 0; v < V; ++v) xf[v] = in ? xf[v] : 0.f;
#pragma unroll
          for (int p = 0; p < P; ++p)
#pragma unroll
            for (int kw = 0; kw < KW; ++kw)
              if (p * SW + kw * DW == j) {
                dw_fma<V>(acc[p], xf, wv[kw]);
              }
        }
      } else {
        for (int kw = 0; kw < a.kW; ++kw) {
          float wv[V];
          dw_weights<V>(wtap + kw * cbv, a.cb, wv);
#pragma unroll
          for (int p = 0; p < P; ++p) {
            const int iw = (ow0 + p) * a.sw - a.pw + kw * a.dw;
            if (static_cast<unsigned>(iw) >= static_cast<unsigned>(a.W)) continue;
            const Vec raw = __ldg(reinterpret_cast<const Vec*>(xrow + static_cast<long long>(iw) * a.C));
            float xv[V];
            dw_unpack<T, V>(raw, xv);
            dw_fma<V>(acc[p], xv, wv);
          }
        }
      }
    }
  }

  T* yrow = y + (((n * a.Do + od) * a.Ho + oh) * static_cast<long long>(a.Wo)) * a.C + c0;
#pragma unroll
  for (int p = 0; p < P; ++p) {
    if (ow0 + p >= a.Wo) break;
    Vec out;
    T* e = reinterpret_cast<T*>(&out);
#pragma unroll
    for (int v = 0; v < V; ++v) e[v] = from_f32<T>(acc[p][v]);
    *reinterpret_cast<Vec*>(yrow + static_cast<long long>(ow0 + p) * a.C) = out;
  }
}

// ---------------------------------------------------------------- TMA-staged form
//
// Persistent CTAs, each bound to one channel tile of CB = cb*4 channels (its
// filters stay in shared memory for the whole launch), walk a static list of
// output tiles of TH x TW pixels of one (n, od).  A tile's input is, per valid
// kd, one slab of span_h x span_w pixels x CB channels, which one TMA tiled
// load brings into shared memory (the hardware zero-fills what lies in the
// padding).  A producer warp keeps a ring of `stages` slabs ahead of eight or
// twelve consumer warps (full / empty mbarriers).  CTA b serves channel tile b % nct
// and tiles b / nct, b / nct + gridDim.x / nct, ...
//
// A consumer thread owns 4 channels (one 8-byte vector for 16-bit types, 16
// bytes for f32) of a block of R output rows x P output columns; consecutive
// threads take consecutive channel vectors of a block, so each slab read of
// a warp is one contiguous run.  The tile is BR x BC blocks (TH = BR*R,
// TW = BC*P).  Products accumulate in fp32 through packed two-lane FMAs.
//
// The consumer forms (kDwSquare, kDwRows, kDwGeneric below) differ in how
// much of the filter sits in registers; in the first two, each input vector a
// thread reads is converted to fp32 once and applied to every (output row,
// output column, tap) that uses it, the pairing resolved at compile time.

struct DwTmaArgs {
  DwArgs d;              // geometry; d.cb = channel vectors (of 4) per tile
  int BR, BC;            // blocks per tile: rows, columns
  int TH, TW;            // tile rows / columns (BR*R, BC*P)
  int span_h, span_w;    // input slab rows / columns
  int tiles_h, tiles_w;  // tiles per output plane
  int nct;               // channel tiles
  int stages;
  int tiles;             // N * Do * tiles_h * tiles_w (below 2^31)
  uint32_t slab_bytes;   // span_h * span_w * cb * vector bytes
  uint32_t slab_pitch;   // slab_bytes rounded up to 128
  uint32_t w_off;        // byte offset of the filters (after the slabs)
  uint32_t tail_off;     // byte offset of the barriers
  unsigned long long timeout_ns;
  int inject_stall;      // test hook: consumer warp 0 first waits on a barrier nothing arrives at
};

constexpr int kDwTmaMaxStages = 4;
constexpr int kDwTmaP = 4;                           // output columns per block

struct DwTmaTail {
  uint64_t full[kDwTmaMaxStages];
  uint64_t empty[kDwTmaMaxStages];
  uint64_t stall;  // never arrived on (the injected-timeout test waits here)
  volatile int abort_flag;
};

struct DwUnit {
  int n, od, oh0, ow0;
};

__device__ __forceinline__ DwUnit dw_unit(const DwTmaArgs& a, int t) {
  DwUnit r;
  r.ow0 = (t % a.tiles_w) * a.TW;
  t /= a.tiles_w;
  r.oh0 = (t % a.tiles_h) * a.TH;
  t /= a.tiles_h;
  r.od = t % a.d.Do;
  r.n = t / a.d.Do;
  return r;
}

// Filters of channel tile `ct` into s_w (layout of dw_widx<V>), by threads
// [tid, tid + count) of the block.
template <typename T, int V>
__device__ __forceinline__ void dw_fill_filters(float* s_w, const DwArgs& g, int ct, int taps, int tid,
                                                int count) {
  const int cbv = g.cb * V;
  const int cbase = ct * cbv;
  for (int i = tid; i < cbv * taps; i += count) {
    const int cl = i / taps;
    const int t = i - cl * taps;
    const int c = cbase + cl;
    s_w[dw_widx<V>(g.flip ? taps - 1 - t : t, cl, g.cb)] =
        c < g.C ? to_f32<T>(static_cast<const T*>(g.w)[static_cast<long long>(c) * taps + t]) : 0.f;
  }
}

// Four channels of T as one vector (8 bytes for 16-bit types, 16 for f32).
template <typename T>
struct DwVec4;
template <>
struct DwVec4<float> {
  using type = float4;
};
template <>
struct DwVec4<__half> {
  using type = uint2;
};
template <>
struct DwVec4<__nv_bfloat16> {
  using type = uint2;
};

__device__ __forceinline__ void dw_unpack4(const float4 r, float2 (&f)[2]) {
  f[0] = make_float2(r.x, r.y);
  f[1] = make_float2(r.z, r.w);
}
template <typename H2, typename U>
__device__ __forceinline__ H2 dw_bits_as(U u) {
  H2 h;
  static_assert(sizeof(H2) == sizeof(U), "size");
  memcpy(&h, &u, sizeof(h));
  return h;
}
__device__ __forceinline__ void dw_unpack4(const uint2 r, float2 (&f)[2], __half) {
  f[0] = __half22float2(dw_bits_as<__half2>(r.x));
  f[1] = __half22float2(dw_bits_as<__half2>(r.y));
}
__device__ __forceinline__ void dw_unpack4(const uint2 r, float2 (&f)[2], __nv_bfloat16) {
  f[0] = __bfloat1622float2(dw_bits_as<__nv_bfloat162>(r.x));
  f[1] = __bfloat1622float2(dw_bits_as<__nv_bfloat162>(r.y));
}
template <typename T>
__device__ __forceinline__ void dw_load4(const uint8_t* p, float2 (&f)[2]) {
  if constexpr (sizeof(T) == 4) {
    dw_unpack4(*reinterpret_cast<const float4*>(p), f);
  } else {
    const uint2 r = *reinterpret_cast<const uint2*>(p);
    dw_unpack4(r, f, T());
  }
}
template <typename T>
__device__ __forceinline__ void dw_store4(T* dst, const float2 (&f)[2]) {
  if constexpr (sizeof(T) == 4) {
    *reinterpret_cast<float4*>(dst) = make_float4(f[0].x, f[0].y, f[1].x, f[1].y);
  } else if constexpr (std::is_same<T, __half>::value) {
    const __half2 a = __float22half2_rn(f[0]), b = __float22half2_rn(f[1]);
    uint2 u;
    memcpy(&u.x, &a, 4);
    memcpy(&u.y, &b, 4);
    *reinterpret_cast<uint2*>(dst) = u;
  } else {
    const __nv_bfloat162 a = __float22bfloat162_rn(f[0]), b = __float22bfloat162_rn(f[1]);
    uint2 u;
    memcpy(&u.x, &a, 4);
    memcpy(&u.y, &b, 4);
    *reinterpret_cast<uint2*>(dst) = u;
  }
}
// The 4 fp32 weights of one tap for one channel vector (layout of dw_widx<4>).
__device__ __forceinline__ void dw_wload4(const float* p, float2 (&w)[2]) {
  const float4 t4 = *reinterpret_cast<const float4*>(p);
  w[0] = make_float2(t4.x, t4.y);
  w[1] = make_float2(t4.z, t4.w);
}
__device__ __forceinline__ void dw_fma4(float2 (&acc)[2], const float2 (&x)[2], const float2 (&w)[2]) {
  acc[0] = __ffma2_rn(x[0], w[0], acc[0]);
  acc[1] = __ffma2_rn(x[1], w[1], acc[1]);
}

// Consumer forms.
//   kDwSquare: K x K filters (K = 3) at width and height stride S, no
//     dilation; all K*K weight vectors of the current kd in registers, blocks
//     of R output rows, every input vector of a block read and converted once.
//   kDwRows: filter width K (5 or 7) at width stride S, no width dilation,
//     any height; one filter row's K weight vectors in registers at a time,
//     R = 1, every input vector of a block row read once per filter row.
//   kDwGeneric: any filter; one slab read per (column, tap).
constexpr int kDwGeneric = 0, kDwSquare = 1, kDwRows = 2;

// CTAs per SM a form is compiled for: the square form (36 weights and 16-64
// accumulators a thread) needs more than half an SM's registers; with twelve
// consumer warps (13 with the producer: at most 4 on each of the SM's four
// schedulers) the limit is 128 registers a thread.  The other forms run two
// CTAs of eight consumer warps.
constexpr int dw_tma_ctas_per_sm(int MODE, int R, int NCW) { return MODE == kDwSquare ? 1 : 2; }

// MODE: consumer form; K, S: its filter width and stride (0 for the generic
// form); R: output rows per block; NCW: consumer warps (warp NCW produces).
template <typename T, int MODE, int K, int S, int R, int NCW>
__global__ void __launch_bounds__(32 * (NCW + 1), dw_tma_ctas_per_sm(MODE, R, NCW))
    conv_fwd_dw_tma_kernel(const __grid_constant__ CUtensorMap tmap_x, const DwTmaArgs a) {
  constexpr int P = kDwTmaP;
  constexpr int VB = 4 * static_cast<int>(sizeof(T));  // bytes per channel vector
  extern __shared__ __align__(128) uint8_t smem[];
  const DwArgs& g = a.d;
  const int taps = g.kD * g.kH * g.kW;
  const int cb = g.cb;
  uint8_t* slabs = smem;
  float* s_w = reinterpret_cast<float*>(smem + a.w_off);
  DwTmaTail* tail = reinterpret_cast<DwTmaTail*>(smem + a.tail_off);
  volatile int* abort_flag = &tail->abort_flag;
  const int warp = static_cast<int>(threadIdx.x >> 5), lane = static_cast<int>(threadIdx.x & 31);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->full[s]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->empty[s]), NCW);
    }
    ptx::mbar_init(ptx::smem_u32(&tail->stall), 1u);
    tail->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == NCW && lane == 0) ptx::prefetch_tmap(&tmap_x);
  ptx::pdl_allow_next();  // setup done: the next launch may start its own
  ptx::pdl_wait_prev();   // the previous launch's writes are visible from here on
  const int ct = static_cast<int>(blockIdx.x) % a.nct;
  const int t_first = static_cast<int>(blockIdx.x) / a.nct, t_step = static_cast<int>(gridDim.x) / a.nct;
  dw_fill_filters<T, 4>(s_w, g, ct, taps, static_cast<int>(threadIdx.x), 32 * (NCW + 1));
  __syncthreads();

  if (warp == NCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long fills = 0;
      bool ok = true;
      for (int t = t_first; ok && t < a.tiles; t += t_step) {
        const DwUnit uc = dw_unit(a, t);
        for (int kd = 0; kd < g.kD; ++kd) {
          const int id = uc.od * g.sd - g.pd + kd * g.dd;
          if (static_cast<unsigned>(id) >= static_cast<unsigned>(g.D)) continue;
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = ptx::smem_u32(&tail->full[stage]);
          ptx::mbar_arrive_expect_tx(fb, a.slab_bytes);
          ptx::tma_load_5d(ptx::smem_u32(slabs + static_cast<size_t>(stage) * a.slab_pitch), &tmap_x, fb,
                           ct * cb * 4, uc.ow0 * g.sw - g.pw, uc.oh0 * g.sh - g.ph, id, uc.n);
          ++fills;
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // every slab issued lands before the CTA's shared memory goes away
        for (int s = 0; s < a.stages; ++s) {
          const long long arms = fills / a.stages + (s < fills % a.stages ? 1 : 0);
          if (arms > 0) wait_drain(ptx::smem_u32(&tail->full[s]), static_cast<uint32_t>((arms - 1) & 1), a.timeout_ns);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = static_cast<int>(threadIdx.x);
  const int cv = tid % cb;
  const int blk = tid / cb;
  const bool blk_active = blk < a.BR * a.BC;
  const int br = blk / a.BC, bc = blk - (blk / a.BC) * a.BC;
  const int c0 = (ct * cb + cv) * 4;
  const bool active = blk_active && c0 < g.C;
  const uint32_t colb = static_cast<uint32_t>(cb) * VB;   // bytes per slab pixel
  const uint32_t rowb = static_cast<uint32_t>(a.span_w) * colb;
  T* __restrict__ y = static_cast<T*>(g.y);
  const float* wbase = s_w + cv * 4;

  // failure-detection test hook: this warp waits, with the short injected
  // limit, on a barrier nothing arrives at; it gives up and raises the abort
  // flag, the other consumers stop at their next wait, the producer drains
  if (a.inject_stall && warp == 0 &&
      !wait_bounded_warp(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected))
    return;

  // register-resident weights of the current kd (square filters)
  float2 wreg[MODE == kDwSquare ? K : 1][MODE == kDwSquare ? K : 1][2];
  int wkd = -1;

  int stage = 0;
  uint32_t phase = 0;
  for (int t = t_first; t < a.tiles; t += t_step) {
    const DwUnit uc = dw_unit(a, t);
    float2 acc[R][P][2];
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
#pragma unroll
      for (int p = 0; p < P; ++p) acc[rr][p][0] = acc[rr][p][1] = make_float2(0.f, 0.f);

    for (int kd = 0; kd < g.kD; ++kd) {
      const int id = uc.od * g.sd - g.pd + kd * g.dd;
      if (static_cast<unsigned>(id) >= static_cast<unsigned>(g.D)) continue;
      if (!wait_bounded_warp(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns, kSiteMmaFull))
        return;
      if (active) {
        const uint8_t* slab = slabs + static_cast<size_t>(stage) * a.slab_pitch + static_cast<uint32_t>(cv) * VB;
        if constexpr (MODE == kDwSquare) {
          if (kd != wkd) {
#pragma unroll
            for (int kh = 0; kh < K; ++kh)
#pragma unroll
              for (int kw = 0; kw < K; ++kw) dw_wload4(wbase + ((kd * K + kh) * K + kw) * cb * 4, wreg[kh][kw]);
            wkd = kd;
          }
          constexpr int RIN = (R - 1) * S + K;
          constexpr int SPAN = (P - 1) * S + K;
          const uint8_t* bp = slab + static_cast<uint32_t>(br * R * S) * rowb + static_cast<uint32_t>(bc * P * S) * colb;
#pragma unroll
          for (int i = 0; i < RIN; ++i) {
#pragma unroll
            for (int j = 0; j < SPAN; ++j) {
              float2 xf[2];
              dw_load4<T>(bp + static_cast<uint32_t>(i) * rowb + static_cast<uint32_t>(j) * colb, xf);
#pragma unroll
              for (int rr = 0; rr < R; ++rr)
#pragma unroll
                for (int kh = 0; kh < K; ++kh)
                  if (rr * S + kh == i) {
#pragma unroll
                    for (int p = 0; p < P; ++p)
#pragma unroll
                      for (int kw = 0; kw < K; ++kw)
                        if (p * S + kw == j) dw_fma4(acc[rr][p], xf, wreg[kh][kw]);
                  }
            }
          }
        } else if constexpr (MODE == kDwRows) {
          constexpr int SPAN = (P - 1) * S + K;
          const uint8_t* bp = slab + static_cast<uint32_t>(br * g.sh) * rowb + static_cast<uint32_t>(bc * P * S) * colb;
          for (int kh = 0; kh < g.kH; ++kh) {
            const uint8_t* rowp = bp + static_cast<uint32_t>(kh * g.dh) * rowb;
            float2 wv[K][2];
#pragma unroll
            for (int kw = 0; kw < K; ++kw) dw_wload4(wbase + ((kd * g.kH + kh) * K + kw) * cb * 4, wv[kw]);
#pragma unroll
            for (int j = 0; j < SPAN; ++j) {
              float2 xf[2];
              dw_load4<T>(rowp + static_cast<uint32_t>(j) * colb, xf);
#pragma unroll
              for (int p = 0; p < P; ++p)
#pragma unroll
                for (int kw = 0; kw < K; ++kw)
                  if (p * S + kw == j) dw_fma4(acc[0][p], xf, wv[kw]);
            }
          }
        } else {
          const uint8_t* bp = slab + static_cast<uint32_t>(br * g.sh) * rowb;
          for (int kh = 0; kh < g.kH; ++kh) {
            const uint8_t* rowp = bp + static_cast<uint32_t>(kh * g.dh) * rowb;
            for (int kw = 0; kw < g.kW; ++kw) {
              float2 wv[2];
              dw_wload4(wbase + ((kd * g.kH + kh) * g.kW + kw) * cb * 4, wv);
#pragma unroll
              for (int p = 0; p < P; ++p) {
                const int col = (bc * P + p) * g.sw + kw * g.dw;
                float2 xf[2];
                dw_load4<T>(rowp + static_cast<uint32_t>(col) * colb, xf);
                dw_fma4(acc[0][p], xf, wv);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&tail->empty[stage]));
      if (++stage == a.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }

    if (active) {
#pragma unroll
      for (int rr = 0; rr < R; ++rr) {
        const int oh = uc.oh0 + br * R + rr;
        if (oh >= g.Ho) break;
        T* yrow = y + ((static_cast<long long>(uc.n) * g.Do + uc.od) * g.Ho + oh) * static_cast<long long>(g.Wo) * g.C + c0;
#pragma unroll
        for (int p = 0; p < P; ++p) {
          const int ow = uc.ow0 + bc * P + p;
          if (ow >= g.Wo) break;
          dw_store4<T>(yrow + static_cast<long long>(ow) * g.C, acc[rr][p]);
        }
      }
    }
  }
}

}  // namespace convfwd
