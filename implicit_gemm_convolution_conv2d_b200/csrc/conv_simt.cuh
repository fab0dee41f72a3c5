// conv_simt.cuh -- fp32 FFMA implicit-GEMM convolution forward (any geometry).
//
// The same GEMM view as the tensor-core kernel (rows = output pixels, columns
// = output channels of one group, reduction over (kd, kh, kw, c) in weight
// order), computed with fp32 fused multiply-adds on the SIMT pipes.  It is the
// path for fp32 tensors: TF32 tensor cores would round every input to 10
// mantissa bits, far outside a 1e-5 relative bound.
//
// Tiles of (16*TM) pixels x (16*TN) channels x 16 K per step, 256 threads.
// Each 16-wide K step is summed into a fresh partial that is then added to the
// running total (two-level summation), which bounds the rounding error by
// about (16 + K/16) units in the last place of sum|x*w| instead of K.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"  // programmatic dependent launch

namespace convfwd {

struct SimtArgs {
  int N, D, H, W, C, O;
  int kD, kH, kW;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  int G, Cg, Og;
  int Do, Ho, Wo;
  long long M;
  int K;
  int flip;   // 1: the filter is read reversed in every spatial dimension
  int taps;   // kD*kH*kW
  int idd, idh, idw;  // input dilation: position z holds x[z / id*] when id* divides z, else 0
  int wtrans;         // 1: w is stored [G*Cg][taps][Og] (a transposed convolution's weights)
  const void* x;
  const void* w;
  void* y;
};

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

constexpr int kSimtBK = 16, kSimtThreads = 256;

// Thread (ty, tx) of a 16 x 16 grid owns output rows (pixels) ty*TM .. ty*TM+TM-1
// of the tile and output channels tx + 16*j, j < TN; the tile is BM = 16*TM
// pixels x BN = 16*TN channels.  BN is chosen on the host to fit O/G (32, 64,
// 80, 96 or 128), so layers like O = 65 or 21 do not compute mostly padding.
// Loads of the next K step go to registers before the current step's FMAs and
// to the other shared-memory buffer after them: one barrier per step.
// Input position z of a dimension dilated by s: true, with z replaced by the
// element index, when the position holds an input element (s = 1: plain bounds).
__device__ __forceinline__ bool simt_undilate(int& z, int s, int n) {
  if (s == 1) return static_cast<unsigned>(z) < static_cast<unsigned>(n);
  if (z < 0 || z % s != 0) return false;
  z /= s;
  return z < n;
}

// TR: the transposed-convolution form (input dilation, transposed weight
// layout), a separate instantiation so the forward kernel is unchanged.
// MASK (forward form, at most 32 filter taps): each loader row keeps a bit
// mask of the taps whose input position lies inside the input and the offset
// of its window origin, so an element costs a mask test and one add instead
// of three bounds checks and an index product.
template <typename T, int TM, int TN, bool TR = false, bool MASK = false>
__global__ void __launch_bounds__(kSimtThreads) conv_fwd_simt_kernel(const SimtArgs a) {
  constexpr int BM = 16 * TM, BN = 16 * TN;
  // Row strides of BM + 2 and BN + 2 floats (twice an odd number): the loader's
  // stores (K row kl = lane & 15 of the warp, pixel / channel lr + 16 i with
  // lr = lane >> 4) then fall in 32 distinct banks; with a stride that is a
  // multiple of 4, rows kl and kl + 8 shared banks (2-way conflicts on every
  // store).  The pixel reads are float2 pairs (8-byte aligned rows).
  static_assert(((BM + 2) / 2) % 2 == 1 && ((BN + 2) / 2) % 2 == 1, "row strides must be 2 x odd");
  static_assert(TM % 2 == 0, "pixel reads are float2 pairs");
  __shared__ __align__(16) float As[2][kSimtBK][BM + 2];
  __shared__ __align__(16) float Bs[2][kSimtBK][BN + 2];

  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ w = static_cast<const T*>(a.w);
  T* __restrict__ y = static_cast<T*>(a.y);
  // (no early trigger: several blocks of this kernel share an SM, and blocks of
  // the next launch waiting beside them slow them down; the next launch starts
  // as these blocks exit)
  ptx::pdl_wait_prev();  // the previous launch's writes are visible from here on

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const long long m0 = static_cast<long long>(blockIdx.x) * BM;
  const int n0 = blockIdx.y * BN;
  const int g = blockIdx.z;

  // loader roles: K element kl = tid & 15 of rows (tid >> 4) + 16 i
  const int kl = tid & 15, lr = tid >> 4;
  bool rvalid[TM];
  long long rbase[TM];
  int rd0[TM], rh0[TM], rw0[TM];
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const long long m = m0 + lr + 16 * i;
    rvalid[i] = m < a.M;
    const long long mm = rvalid[i] ? m : 0;
    const int ow = static_cast<int>(mm % a.Wo);
    long long q = mm / a.Wo;
    const int oh = static_cast<int>(q % a.Ho);
    q /= a.Ho;
    const int od = static_cast<int>(q % a.Do);
    const long long n = q / a.Do;
    rbase[i] = n * a.D * a.H * a.W * static_cast<long long>(a.C) + static_cast<long long>(g) * a.Cg;
    rd0[i] = od * a.sd - a.pd;
    rh0[i] = oh * a.sh - a.ph;
    rw0[i] = ow * a.sw - a.pw;
  }
  // MASK: the window origin of each loader row (possibly outside the input) as
  // an element offset, and the taps that land inside the input
  long long rorg[MASK ? TM : 1];
  uint32_t rmask[MASK ? TM : 1];
  if constexpr (MASK) {
#pragma unroll
    for (int i = 0; i < TM; ++i) {
      rorg[i] = rbase[i] + ((static_cast<long long>(rd0[i]) * a.H + rh0[i]) * a.W + rw0[i]) * a.C;
      uint32_t msk = 0;
      int t = 0;
      for (int kd = 0; kd < a.kD; ++kd)
        for (int kh = 0; kh < a.kH; ++kh)
          for (int kw = 0; kw < a.kW; ++kw, ++t) {
            const int zd = rd0[i] + kd * a.dd, zh = rh0[i] + kh * a.dh, zw = rw0[i] + kw * a.dw;
            if (static_cast<unsigned>(zd) < static_cast<unsigned>(a.D) &&
                static_cast<unsigned>(zh) < static_cast<unsigned>(a.H) &&
                static_cast<unsigned>(zw) < static_cast<unsigned>(a.W))
              msk |= 1u << t;
          }
      rmask[i] = rvalid[i] ? msk : 0u;
    }
  }
  const T* wrow[TN];
  bool ovalid[TN];
#pragma unroll
  for (int j = 0; j < TN; ++j) {
    const int o = n0 + lr + 16 * j;
    ovalid[j] = o < a.Og;
    wrow[j] = w + static_cast<long long>(g * a.Og + (ovalid[j] ? o : 0)) * a.K;
  }
  // carried decode of k = k0 + kl into (kd, kh, kw, c)
  int c = kl, kw = 0, kh = 0, kd = 0;
  while (c >= a.Cg) {
    c -= a.Cg;
    if (++kw == a.kW) { kw = 0; if (++kh == a.kH) { kh = 0; ++kd; } }
  }

  float ra[TM], rb[TN];
  const auto load_step = [&](int k0) {
    const int k = k0 + kl;
    const bool kv = k < a.K;
    const int id = kd * a.dd, ih = kh * a.dh, iw = kw * a.dw;
    if constexpr (MASK) {
      const int tapk = (kd * a.kH + kh) * a.kW + kw;
      const long long toff = (static_cast<long long>(id) * a.H + ih) * static_cast<long long>(a.W) * a.C +
                             static_cast<long long>(iw) * a.C + c;
      const uint32_t bit = kv ? (1u << tapk) : 0u;
#pragma unroll
      for (int i = 0; i < TM; ++i) ra[i] = (rmask[i] & bit) ? to_f32<T>(x[rorg[i] + toff]) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < (MASK ? 0 : TM); ++i) {
      float v = 0.f;
      int zd = rd0[i] + id, zh = rh0[i] + ih, zw = rw0[i] + iw;
      bool in;
      if constexpr (TR) {
        in = simt_undilate(zd, a.idd, a.D) && simt_undilate(zh, a.idh, a.H) && simt_undilate(zw, a.idw, a.W);
      } else {
        in = static_cast<unsigned>(zd) < static_cast<unsigned>(a.D) &&
             static_cast<unsigned>(zh) < static_cast<unsigned>(a.H) &&
             static_cast<unsigned>(zw) < static_cast<unsigned>(a.W);
      }
      if (rvalid[i] && kv && in)
        v = to_f32<T>(x[rbase[i] + ((static_cast<long long>(zd) * a.H + zh) * a.W + zw) * a.C + c]);
      ra[i] = v;
    }
    // the weight element: k itself, or with flip the mirrored tap's channel c;
    // transposed storage [G*Cg][taps][Og] puts it at ((g*Cg + c)*taps + tap)*Og + o
    const int tapk = (kd * a.kH + kh) * a.kW + kw;
    const int wt = a.flip ? a.taps - 1 - tapk : tapk;
    if (TR && a.wtrans) {
      const long long wb = (static_cast<long long>(g * a.Cg + c) * a.taps + wt) * a.Og;
#pragma unroll
      for (int j = 0; j < TN; ++j) rb[j] = (ovalid[j] && kv) ? to_f32<T>(w[wb + n0 + lr + 16 * j]) : 0.f;
    } else {
      const int wk = wt * a.Cg + c;
#pragma unroll
      for (int j = 0; j < TN; ++j) rb[j] = (ovalid[j] && kv) ? to_f32<T>(wrow[j][wk]) : 0.f;
    }
    // advance the carried decode by one K step
    c += kSimtBK;
    while (c >= a.Cg) {
      c -= a.Cg;
      if (++kw == a.kW) { kw = 0; if (++kh == a.kH) { kh = 0; ++kd; } }
    }
  };
  const auto store_step = [&](int buf) {
#pragma unroll
    for (int i = 0; i < TM; ++i) As[buf][kl][lr + 16 * i] = ra[i];
#pragma unroll
    for (int j = 0; j < TN; ++j) Bs[buf][kl][lr + 16 * j] = rb[j];
  };

  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

  load_step(0);
  store_step(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < a.K; k0 += kSimtBK) {
    const bool more = k0 + kSimtBK < a.K;
    if (more) load_step(k0 + kSimtBK);  // global loads in flight during the FMAs below
    float part[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) part[i][j] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kSimtBK; ++kk) {
      float ar[TM], br[TN];
#pragma unroll
      for (int i = 0; i < TM; i += 2) {
        const float2 v = *reinterpret_cast<const float2*>(&As[buf][kk][ty * TM + i]);
        ar[i] = v.x;
        ar[i + 1] = v.y;
      }
#pragma unroll
      for (int j = 0; j < TN; ++j) br[j] = Bs[buf][kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) part[i][j] = fmaf(ar[i], br[j], part[i][j]);
    }
    // two-level summation: each 16-wide K step is summed apart, then added
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] += part[i][j];
    if (more) {
      store_step(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }

#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const long long m = m0 + ty * TM + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int o = n0 + tx + 16 * j;
      if (o < a.Og) y[m * a.O + static_cast<long long>(g) * a.Og + o] = from_f32<T>(acc[i][j]);
    }
  }
}

}  // namespace convfwd
