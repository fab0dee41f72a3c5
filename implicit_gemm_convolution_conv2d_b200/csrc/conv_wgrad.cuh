// conv_wgrad.cuh -- weight gradient of the convolution forward pass.
//
// For the forward pass y = conv(x, w) (channels-last, stride / padding /
// dilation / groups as in conv_fwd), the gradient of its weights given the
// gradient dy of its output is
//   dw[o, kd, kh, kw, c] = sum over pixels (n, od, oh, ow) of
//       dy[n, od, oh, ow, o] * x[n, od*sd - pd + kd*dd, oh*sh - ph + kh*dh,
//                                ow*sw - pw + kw*dw, g*Cg + c]
// (x = 0 outside the input): per group an implicit GEMM with M = Og output
// channels, N = taps*Cg weight columns and a reduction over the P = N*Do*Ho*Wo
// output pixels, its B operand being the im2col matrix of x read in place.
//
// FP32 FMA kernel: a block computes a 64 x 64 tile of one group's dw over one
// contiguous range of pixels (split-K across blocks) and stores that partial
// tile, in fp32, into its own slice of a workspace [split][O][taps*Cg]; a
// second kernel adds the slices of every element in split order and rounds
// the sum to the output type.  No atomics: the result does not depend on the
// order in which blocks run.  Each 16-pixel K step stages dy (16 x 64 output
// channels) and the im2col rows (16 x 64 weight columns) in shared memory as
// fp32; a thread owns 4 x 4 outputs, which it sums in three levels (a K step
// into a fresh partial, 16 steps into a segment, segments into the total) so
// that rounding grows with the number of terms per level, not with the
// length of the range.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "conv_simt.cuh"  // to_f32 / from_f32

namespace convfwd {

struct WgArgs {
  int N, D, H, W, C, O;
  int kD, kH, kW;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  int pd_hi, ph_hi, pw_hi;  // padding above each dimension
  int G, Cg, Og;
  int Do, Ho, Wo;
  int taps, ncols;   // kD*kH*kW, taps*Cg
  long long P;       // output pixels N*Do*Ho*Wo (the reduction length)
  long long chunk;   // pixels per split, a multiple of 16
  int nsplit;        // splits of the reduction (gridDim.z = G * nsplit)
  const void* x;
  const void* dy;
  float* part;       // [nsplit][O][taps*Cg] fp32 partial sums (every element written)
};

constexpr int kWgBM = 64, kWgBN = 64, kWgBK = 16, kWgThreads = 256;
constexpr int kWgSegSteps = 16;  // K steps per segment of the three-level sum

template <typename T>
__global__ void __launch_bounds__(kWgThreads) conv_wgrad_kernel(const WgArgs a) {
  __shared__ __align__(16) float As[kWgBK][kWgBM + 4];  // dy: [pixel][output channel]
  __shared__ __align__(16) float Bs[kWgBK][kWgBN + 4];  // im2col of x: [pixel][weight column]

  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ dy = static_cast<const T*>(a.dy);
  // (no early trigger: several blocks of this kernel share an SM, and blocks of
  // the next launch waiting beside them slow them down; the next launch starts
  // as these blocks exit)
  ptx::pdl_wait_prev();  // the previous launch's writes are visible from here on
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int col0 = blockIdx.x * kWgBN;
  const int o0 = blockIdx.y * kWgBM;
  const int g = blockIdx.z / a.nsplit;
  const int split = blockIdx.z - g * a.nsplit;
  const long long p_begin = static_cast<long long>(split) * a.chunk;
  const long long p_end = min(a.P, p_begin + a.chunk);

  // loader roles: pixel row kk = ty of the K step, 4 consecutive columns
  // (output channels for A, weight columns for B) starting at tx*4
  const int kk = ty;
  int bkd[4], bkh[4], bkw[4], bc[4];
  bool bvalid[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int col = col0 + tx * 4 + j;
    bvalid[j] = col < a.ncols;
    const int cc = bvalid[j] ? col : 0;
    const int tap = cc / a.Cg;
    bc[j] = cc - tap * a.Cg;
    bkw[j] = tap % a.kW;
    bkh[j] = (tap / a.kW) % a.kH;
    bkd[j] = tap / (a.kW * a.kH);
  }

  float acc[4][4], seg[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = seg[i][j] = 0.f;

  int nstep = 0;
  for (long long p0 = p_begin; p0 < p_end; p0 += kWgBK) {
    const long long p = p0 + kk;
    const bool pv = p < p_end;
    int n = 0, od = 0, oh = 0, ow = 0;
    if (pv) {
      long long q = p;
      ow = static_cast<int>(q % a.Wo);
      q /= a.Wo;
      oh = static_cast<int>(q % a.Ho);
      q /= a.Ho;
      od = static_cast<int>(q % a.Do);
      n = static_cast<int>(q / a.Do);
    }
    // A: dy[p, g*Og + o0 + tx*4 + j]
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = o0 + tx * 4 + j;
      As[kk][tx * 4 + j] = (pv && o < a.Og) ? to_f32<T>(dy[p * a.O + static_cast<long long>(g) * a.Og + o]) : 0.f;
    }
    // B: x at the pixel's input position shifted by each column's tap
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v = 0.f;
      if (pv && bvalid[j]) {
        const int id = od * a.sd - a.pd + bkd[j] * a.dd;
        const int ih = oh * a.sh - a.ph + bkh[j] * a.dh;
        const int iw = ow * a.sw - a.pw + bkw[j] * a.dw;
        if (static_cast<unsigned>(id) < static_cast<unsigned>(a.D) &&
            static_cast<unsigned>(ih) < static_cast<unsigned>(a.H) &&
            static_cast<unsigned>(iw) < static_cast<unsigned>(a.W))
          v = to_f32<T>(x[((((static_cast<long long>(n) * a.D + id) * a.H + ih) * a.W + iw) * a.C) +
                          static_cast<long long>(g) * a.Cg + bc[j]]);
      }
      Bs[kk][tx * 4 + j] = v;
    }
    __syncthreads();
    float st[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) st[i][j] = 0.f;
#pragma unroll
    for (int k = 0; k < kWgBK; ++k) {
      const float4 av = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) st[i][j] = fmaf(ar[i], br[j], st[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) seg[i][j] += st[i][j];
    if (++nstep == kWgSegSteps) {
      nstep = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] += seg[i][j];
          seg[i][j] = 0.f;
        }
    }
    __syncthreads();
  }

  float* __restrict__ part = a.part + static_cast<long long>(split) * a.O * a.ncols;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int o = o0 + ty * 4 + i;
    if (o >= a.Og) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = col0 + tx * 4 + j;
      if (col < a.ncols) part[static_cast<long long>(g * a.Og + o) * a.ncols + col] = acc[i][j] + seg[i][j];
    }
  }
}

// dw[i] = the sum of the nsplit partial slices of element i, added in split
// order in fp32, rounded to nearest in the output type.
template <typename T>
__global__ void __launch_bounds__(256) conv_wgrad_reduce_kernel(const float* __restrict__ part, T* __restrict__ dw,
                                                                long long n, int nsplit) {
  const long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  ptx::pdl_wait_prev();  // the ranges' partial sums are complete and visible
  if (i >= n) return;
  float s = part[i];
  for (int k = 1; k < nsplit; ++k) s += part[static_cast<long long>(k) * n + i];
  dw[i] = from_f32<T>(s);
}

// The same for four consecutive elements a thread (n % 4 == 0, slices
// 16-byte aligned): 16-byte loads of the slices, one 8- or 16-byte store.
template <typename T>
__global__ void __launch_bounds__(256) conv_wgrad_reduce4_kernel(const float* __restrict__ part, T* __restrict__ dw,
                                                                 long long n, int nsplit) {
  const long long i = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) * 4;
  ptx::pdl_wait_prev();  // the ranges' partial sums are complete and visible
  if (i >= n) return;
  float4 s = *reinterpret_cast<const float4*>(part + i);
  for (int k = 1; k < nsplit; ++k) {
    const float4 v = *reinterpret_cast<const float4*>(part + static_cast<long long>(k) * n + i);
    s.x += v.x;
    s.y += v.y;
    s.z += v.z;
    s.w += v.w;
  }
  if constexpr (sizeof(T) == 4) {
    *reinterpret_cast<float4*>(dw + i) = s;
  } else {
    T o[4] = {from_f32<T>(s.x), from_f32<T>(s.y), from_f32<T>(s.z), from_f32<T>(s.w)};
    *reinterpret_cast<uint2*>(dw + i) = *reinterpret_cast<const uint2*>(o);
  }
}

}  // namespace convfwd
