// conv_simt.cuh -- fp32 FFMA implicit-GEMM convolution forward (any geometry).
//
// The same GEMM view as the tensor-core kernel (rows = output pixels, columns
// = output channels of one group, reduction over (kd, kh, kw, c) in weight
// order), computed with fp32 fused multiply-adds on the SIMT pipes.  It is the
// path for fp32 tensors: TF32 tensor cores would round every input to 10
// mantissa bits, far outside a 1e-5 relative bound.
//
// Tile 64 pixels x 64 channels x 16 K per step, 256 threads, 4x4 outputs per
// thread.  Each 16-wide K step is summed into a fresh partial that is then
// added to the running total (two-level summation), which bounds the rounding
// error by about (16 + K/16) units in the last place of sum|x*w| instead of K.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace convfwd {

struct SimtArgs {
  int N, D, H, W, C, O;
  int kD, kH, kW;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  int G, Cg, Og;
  int Do, Ho, Wo;
  long long M;
  int K;
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

constexpr int kSimtBM = 64, kSimtBN = 64, kSimtBK = 16, kSimtThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) conv_fwd_simt_kernel(const SimtArgs a) {
  __shared__ __align__(16) float As[kSimtBK][kSimtBM + 4];
  __shared__ __align__(16) float Bs[kSimtBK][kSimtBN + 4];

  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ w = static_cast<const T*>(a.w);
  T* __restrict__ y = static_cast<T*>(a.y);

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const long long m0 = static_cast<long long>(blockIdx.x) * kSimtBM;
  const int n0 = blockIdx.y * kSimtBN;
  const int g = blockIdx.z;

  // loader roles: element (kl, row) with kl = tid & 15, row = (tid >> 4) + 16 i
  const int kl = tid & 15;
  bool rvalid[4];
  long long rbase[4];
  int rd0[4], rh0[4], rw0[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long m = m0 + (tid >> 4) + 16 * i;
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
  // carried decode of k = k0 + kl into (kd, kh, kw, c)
  int c = kl, kw = 0, kh = 0, kd = 0;
  while (c >= a.Cg) {
    c -= a.Cg;
    if (++kw == a.kW) { kw = 0; if (++kh == a.kH) { kh = 0; ++kd; } }
  }

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < a.K; k0 += kSimtBK) {
    const int k = k0 + kl;
    // A tile
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = 0.f;
      if (rvalid[i] && k < a.K) {
        const int id = rd0[i] + kd * a.dd, ih = rh0[i] + kh * a.dh, iw = rw0[i] + kw * a.dw;
        if (static_cast<unsigned>(id) < static_cast<unsigned>(a.D) &&
            static_cast<unsigned>(ih) < static_cast<unsigned>(a.H) &&
            static_cast<unsigned>(iw) < static_cast<unsigned>(a.W))
          v = to_f32<T>(x[rbase[i] + ((static_cast<long long>(id) * a.H + ih) * a.W + iw) * a.C + c]);
      }
      As[kl][(tid >> 4) + 16 * i] = v;
    }
    // B tile
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int o = n0 + (tid >> 4) + 16 * i;
      float v = 0.f;
      if (o < a.Og && k < a.K)
        v = to_f32<T>(w[static_cast<long long>(g * a.Og + o) * a.K + k]);
      Bs[kl][(tid >> 4) + 16 * i] = v;
    }
    __syncthreads();

    float part[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kSimtBK; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(ar[i], br[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
    __syncthreads();

    // advance the carried decode by one K step
    c += kSimtBK;
    while (c >= a.Cg) {
      c -= a.Cg;
      if (++kw == a.kW) { kw = 0; if (++kh == a.kH) { kh = 0; ++kd; } }
    }
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = n0 + tx * 4 + j;
      if (o < a.Og) y[m * a.O + static_cast<long long>(g) * a.Og + o] = from_f32<T>(acc[i][j]);
    }
  }
}

}  // namespace convfwd
