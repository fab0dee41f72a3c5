// conv_fwd.cu -- the C ABI (include/conv_fwd.h): argument checks, kernel
// choice and tiling, TMA tensor-map encoding, launches.  Nothing here touches
// tensor data; every step of the convolution runs in the kernels of
// conv_tc.cuh (f16/bf16, tcgen05 tensor cores) and conv_simt.cuh (f32).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <numeric>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/conv_fwd.h"
#include "conv_halo.cuh"
#include "conv_simt.cuh"
#include "conv_tc.cuh"
#include "conv_tct.cuh"
#include "conv_halo_t.cuh"
#include "conv_phase.cuh"
#include "conv_dw.cuh"
#include "conv_staged.cuh"
#include "conv_wgrad.cuh"
#include "launch.cuh"
#include "conv_wgrad_tc.cuh"
#include "conv_tconv.cuh"

namespace convfwd {
namespace {

constexpr int kVersion = 100;                       // 0.1.0
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s per pipeline wait
constexpr uint32_t kSmemBudget = 227 * 1024;        // max dynamic smem per CTA on sm_100
constexpr int kMaxDevices = 64;
constexpr long long kMaxResidentB = 96 * 1024;              // weights kept in smem by the gather kernel

struct Problem {
  int N, D, H, W, C, O, kD, kH, kW;
  int s[3], p[3], d[3];  // p: padding below each dimension (the index origin is -p)
  int p_hi[3];           // padding above each dimension (sets the output extent with p)
  int flip;              // 1: the filter is read reversed in every spatial dimension
  int idil[3];           // input dilation (a transposed convolution's stride); 1 = none
  int wtrans;            // 1: w is stored [G*Cg][taps][Og] (a transposed convolution's weights)
  int G, Cg, Og;
  int Do, Ho, Wo;
  long long M;
  long long K;
  int dtype;
  size_t esize;
  size_t x_bytes, w_bytes, y_bytes;
};

long long extent(long long in, int k, int s, int p_lo, int p_hi, int d) {
  const long long num = in + static_cast<long long>(p_lo) + p_hi - static_cast<long long>(d) * (k - 1) - 1;
  if (num < 0) return 0;
  return num / s + 1;
}

int out_dims_impl(int D, int H, int W, int kD, int kH, int kW, const int stride[3], const int pad_lo[3],
                  const int pad_hi[3], const int dil[3], int out[3]) {
  if (!stride || !pad_lo || !pad_hi || !dil || !out) return CONV_EINVAL;
  const int in[3] = {D, H, W};
  const int k[3] = {kD, kH, kW};
  for (int i = 0; i < 3; ++i) {
    if (in[i] <= 0 || k[i] <= 0 || stride[i] <= 0 || dil[i] <= 0 || pad_lo[i] < 0 || pad_hi[i] < 0)
      return CONV_EINVAL;
    const long long e = extent(in[i], k[i], stride[i], pad_lo[i], pad_hi[i], dil[i]);
    if (e <= 0 || e > 0x7fffffffLL) return CONV_EINVAL;
    out[i] = static_cast<int>(e);
  }
  return CONV_OK;
}

bool mul_ok(long long a, long long b, long long& r) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > (1LL << 62) / a) return false;
  r = a * b;
  return true;
}

int make_problem(Problem& P, int N, int D, int H, int W, int C, int O, int kD, int kH, int kW,
                 const int stride[3], const int pad_lo[3], const int pad_hi[3], const int dil[3], int groups,
                 int flip, int dtype) {
  if (dtype != CONV_F32 && dtype != CONV_F16 && dtype != CONV_BF16) return CONV_EDTYPE;
  if (N <= 0 || C <= 0 || O <= 0 || groups <= 0) return CONV_EINVAL;
  if (C % groups != 0 || O % groups != 0) return CONV_EINVAL;
  if (flip != 0 && flip != 1) return CONV_EINVAL;
  int out[3];
  const int rc = out_dims_impl(D, H, W, kD, kH, kW, stride, pad_lo, pad_hi, dil, out);
  if (rc != CONV_OK) return rc;
  P.N = N; P.D = D; P.H = H; P.W = W; P.C = C; P.O = O; P.kD = kD; P.kH = kH; P.kW = kW;
  for (int i = 0; i < 3; ++i) {
    P.s[i] = stride[i]; P.p[i] = pad_lo[i]; P.p_hi[i] = pad_hi[i]; P.d[i] = dil[i];
  }
  P.flip = flip;
  P.idil[0] = P.idil[1] = P.idil[2] = 1;
  P.wtrans = 0;
  P.G = groups; P.Cg = C / groups; P.Og = O / groups;
  P.Do = out[0]; P.Ho = out[1]; P.Wo = out[2];
  P.dtype = dtype;
  P.esize = dtype == CONV_F32 ? 4 : 2;
  long long nx, nw, ny, t;
  if (!mul_ok(N, D, t) || !mul_ok(t, H, t) || !mul_ok(t, W, t) || !mul_ok(t, C, nx)) return CONV_EINVAL;
  if (!mul_ok(kD, kH, t) || !mul_ok(t, kW, t) || !mul_ok(t, P.Cg, P.K)) return CONV_EINVAL;
  if (!mul_ok(O, P.K, nw)) return CONV_EINVAL;
  if (!mul_ok(N, P.Do, t) || !mul_ok(t, P.Ho, t) || !mul_ok(t, P.Wo, P.M) || !mul_ok(P.M, O, ny))
    return CONV_EINVAL;
  // kernel-side limits: K, per-row counts and tile counts are 32-bit
  if (P.K > 0x7fffffffLL || P.M > (1LL << 46)) return CONV_EINVAL;
  if (!mul_ok(nx, static_cast<long long>(P.esize), t) || !mul_ok(nw, static_cast<long long>(P.esize), t) ||
      !mul_ok(ny, static_cast<long long>(P.esize), t))
    return CONV_EINVAL;
  P.x_bytes = static_cast<size_t>(nx) * P.esize;
  P.w_bytes = static_cast<size_t>(nw) * P.esize;
  P.y_bytes = static_cast<size_t>(ny) * P.esize;
  return CONV_OK;
}

// Output extents of the transposed convolution: (I-1)*s - 2p + d*(k-1) + 1 + op
// per dimension, op (output padding) in [0, max(s, d)).
int convT_dims_impl(int D, int H, int W, int kD, int kH, int kW, const int stride[3], const int pad[3],
                    const int out_pad[3], const int dil[3], int out[3]) {
  if (!stride || !pad || !out_pad || !dil || !out) return CONV_EINVAL;
  const int in[3] = {D, H, W};
  const int k[3] = {kD, kH, kW};
  for (int i = 0; i < 3; ++i) {
    if (in[i] <= 0 || k[i] <= 0 || stride[i] <= 0 || dil[i] <= 0 || pad[i] < 0 || out_pad[i] < 0)
      return CONV_EINVAL;
    if (out_pad[i] >= stride[i] && out_pad[i] >= dil[i]) return CONV_EINVAL;
    const long long e = (static_cast<long long>(in[i]) - 1) * stride[i] - 2LL * pad[i] +
                        static_cast<long long>(dil[i]) * (k[i] - 1) + 1 + out_pad[i];
    if (e <= 0 || e > 0x7fffffffLL) return CONV_EINVAL;
    out[i] = static_cast<int>(e);
  }
  return CONV_OK;
}

// The transposed convolution of x [N,D,H,W,Cin] by w [Cin,kD,kH,kW,Cout/G] as
// a forward convolution: the input zero-dilated by the stride, stride 1, the
// filter mirrored (flip) with its channel axes exchanged (wtrans), and padding
// d*(k-1) - p below and d*(k-1) - p + op above.  Padding beyond d*(k-1) (a
// crop of the dilated sum) is not supported.
int make_transpose_problem(Problem& P, int N, int D, int H, int W, int Cin, int Cout, int kD, int kH, int kW,
                           const int stride[3], const int pad[3], const int out_pad[3], const int dil[3],
                           int groups, int dtype) {
  int out[3];
  int rc = convT_dims_impl(D, H, W, kD, kH, kW, stride, pad, out_pad, dil, out);
  if (rc != CONV_OK) return rc;
  const int k[3] = {kD, kH, kW};
  int lo[3], hi[3], one[3] = {1, 1, 1};
  for (int i = 0; i < 3; ++i) {
    const long long span = static_cast<long long>(dil[i]) * (k[i] - 1);
    if (pad[i] > span) return CONV_EUNSUPPORTED;
    lo[i] = static_cast<int>(span - pad[i]);
    hi[i] = static_cast<int>(span - pad[i] + out_pad[i]);
  }
  // extents of the zero-dilated input
  long long dd[3];
  const int in[3] = {D, H, W};
  for (int i = 0; i < 3; ++i) {
    dd[i] = (static_cast<long long>(in[i]) - 1) * stride[i] + 1;
    if (dd[i] > 0x7fffffffLL) return CONV_EINVAL;
  }
  rc = make_problem(P, N, static_cast<int>(dd[0]), static_cast<int>(dd[1]), static_cast<int>(dd[2]), Cin, Cout, kD,
                    kH, kW, one, lo, hi, dil, groups, 1, dtype);
  if (rc != CONV_OK) return rc;
  if (P.Do != out[0] || P.Ho != out[1] || P.Wo != out[2]) return CONV_EINVAL;  // (the two extents agree)
  P.D = D; P.H = H; P.W = W;
  for (int i = 0; i < 3; ++i) P.idil[i] = stride[i];
  P.wtrans = 1;
  long long nx, t;
  if (!mul_ok(N, D, t) || !mul_ok(t, H, t) || !mul_ok(t, W, t) || !mul_ok(t, Cin, nx)) return CONV_EINVAL;
  P.x_bytes = static_cast<size_t>(nx) * P.esize;
  return CONV_OK;
}

// Problems every kernel can take: no input dilation, weights in the forward layout.
bool plain_input(const Problem& P) {
  return P.idil[0] == 1 && P.idil[1] == 1 && P.idil[2] == 1 && !P.wtrans;
}

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

int check_pointers(const Problem& P, const void* x, const void* w, const void* y) {
  if (!x || !w || !y) return CONV_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(y)) & 15)
    return CONV_EALIGN;
  if (overlaps(y, P.y_bytes, x, P.x_bytes) || overlaps(y, P.y_bytes, w, P.w_bytes)) return CONV_EALIAS;
  return CONV_OK;
}

// ---------------------------------------------------------------- device info

// Test hook (conv_debug_inject_stall): when non-zero, the next launch of a
// kernel with pipeline waits (the tensor-core kernels, the TMA depthwise
// kernel) makes one of its threads wait on a barrier that nothing arrives at,
// with this limit in nanoseconds, so the kernel's timeout path runs.  One-shot.
std::atomic<unsigned long long> g_inject_stall_ns{0};

struct DeviceInfo {
  bool init = false;
  int sms = 0;
  bool attrs_set = false;
  // CTA pairs that fit on the device at once, per launched pair kernel
  // (index: halo * 2 + bf16), with the dynamic smem each count was measured for
  size_t pair_smem[4] = {0, 0, 0, 0};
  int pair_clusters[4] = {0, 0, 0, 0};
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

int current_device(int& dev) {
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CONV_ELAUNCH;
  return CONV_OK;
}

int device_sms(int dev, int& sms) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev[dev].init) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return CONV_ELAUNCH;
    g_dev[dev].sms = v;
    g_dev[dev].init = true;
  }
  sms = g_dev[dev].sms;
  return CONV_OK;
}

int set_kernel_attrs(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev[dev].attrs_set) return CONV_OK;
  const int bytes = static_cast<int>(kSmemBudget);
  cudaError_t e = cudaSuccess;
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_TMA, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_TMA, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_GATHER, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_GATHER, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_GATHER, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_GATHER, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_GATHER, false, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_kernel<MODE_GATHER, true, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_t_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_t_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_t_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_t_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_t_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_halo_t_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_phase_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_phase_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_wgrad_tc_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_wgrad_tc_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_tconv_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_tconv_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<false, 3, 3, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<false, 3, 3, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<false, 0, 0, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<false, 0, 0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<true, 3, 3, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<true, 3, 3, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<true, 0, 0, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  e = e != cudaSuccess ? e : cudaFuncSetAttribute(conv_fwd_tc_staged_kernel<true, 0, 0, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return CONV_ELAUNCH;
  g_dev[dev].attrs_set = true;
  return CONV_OK;
}

// ---------------------------------------------------------------- driver API

typedef CUresult (*PfnEncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
typedef CUresult (*PfnEncodeIm2col)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const int*, const int*, cuuint32_t, cuuint32_t,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DriverFns {
  bool tried = false;
  PfnEncodeTiled tiled = nullptr;
  PfnEncodeIm2col im2col = nullptr;
  int driver_version = 0;
};
DriverFns g_drv;

const DriverFns& driver_fns() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_drv.tried) {
    g_drv.tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_drv.tiled = reinterpret_cast<PfnEncodeTiled>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeIm2col", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_drv.im2col = reinterpret_cast<PfnEncodeIm2col>(f);
    cudaDriverGetVersion(&g_drv.driver_version);
  }
  return g_drv;
}

// Drivers up to 13.1 mis-encode one descriptor field for tensors under
// 128 KiB; clearing bit 21 of the second 64-bit word is the documented
// remedy used by NVIDIA's CUTLASS (cute/atom/copy_traits_sm90_tma.hpp).
void small_tensor_fixup(CUtensorMap& m, size_t tensor_bytes, int driver_version) {
  if (driver_version <= 13010 && tensor_bytes < 131072) {
    uint64_t* words = reinterpret_cast<uint64_t*>(&m);
    words[1] &= ~(1ull << 21);
  }
}

// ---------------------------------------------------------------- planning

struct TcPlan {
  int variant;
  bool pair;      // CTA-pair (cta_group::2) tiles of 256 rows
  TcArgs args;
  int ctas;
  size_t smem;
};

int round_up(int v, int m) { return (v + m - 1) / m * m; }

// K sub-blocks per pipeline stage.  Every stage costs a fixed barrier-wait /
// MMA-issue / commit round trip (measured on B200 at roughly 700-900 SM
// cycles), which the tensor pipe hides only if one stage carries about as much
// MMA work; one sub-block of kc K-elements is kc/16 MMAs of BN/2 cycles each
// (per SM, M = 128 rows).  Take enough sub-blocks for ~1024 cycles, then
// shrink until at least two stages fit in `avail` bytes.
int choose_kbs(int BN, int kc, uint32_t sub_bytes, long long avail, int max_kbs, int& stages) {
  const int cycles_per_sub = (kc / 16) * (BN / 2);
  int kbs = std::max(1, std::min(max_kbs, (1024 + cycles_per_sub - 1) / cycles_per_sub));
  while (kbs > 1 && avail / (static_cast<long long>(kbs) * sub_bytes) < 2) --kbs;
  stages = static_cast<int>(std::min<long long>(8, avail / (static_cast<long long>(kbs) * sub_bytes)));
  return kbs;
}

uint32_t next_pow2_cols(uint32_t v) {
  uint32_t c = 32;
  while (c < v) c <<= 1;
  return c;
}

// Can the TMA im2col producer describe this problem?  The corner offsets of
// the pixel bounding box and the per-tap offsets must fit the ranges of the
// tensor rank (rank 4: [-128, 127]; rank 5: [-16, 15]); traversal strides
// are at most 8; the pixel rows must be 16-byte strided (C % 8 == 0) and the
// channel chunk a multiple of 16 elements for the MMA K step.
// A 2-D problem: one input plane, one filter plane, and no depth padding on
// either side (the depth extent is then 1).
bool is_2d(const Problem& P) { return P.D == 1 && P.kD == 1 && P.p[0] == 0 && P.p_hi[0] == 0; }

bool tma_fits(const Problem& P, bool& rank5) {
  if (P.dtype == CONV_F32) return false;
  if (P.Cg % 16 != 0) return false;
  rank5 = !is_2d(P);
  const int lo = rank5 ? -16 : -128, hi = rank5 ? 15 : 127;
  const int ks[3] = {P.kD, P.kH, P.kW};
  for (int i = rank5 ? 0 : 1; i < 3; ++i) {
    if (P.s[i] > 8) return false;
    const int lower = -P.p[i];
    const long long upper = static_cast<long long>(P.p_hi[i]) - static_cast<long long>(P.d[i]) * (ks[i] - 1);
    const long long off = static_cast<long long>(P.d[i]) * (ks[i] - 1);
    if (lower < lo || lower > hi || upper < lo || upper > hi || off > hi) return false;
  }
  if (P.N > 0x7fffffff / 2) return false;
  return true;
}

// Can the plain-orientation halo kernel run this problem?  Stride 1, channel
// chunks of 64 or 32, the strip box inside the TMA box limits (256 per
// dimension), rank 4 or 5.
constexpr int kHaloTileH = 16, kHaloTileW = 8;

bool halo_fits(const Problem& P, bool& rank5) {
  if (P.dtype == CONV_F32 || P.Cg % 32 != 0) return false;
  if (P.s[0] != 1 || P.s[1] != 1 || P.s[2] != 1) return false;
  rank5 = !is_2d(P);
  const long long hh = kHaloTileH + static_cast<long long>(P.d[1]) * (P.kH - 1);
  if (hh > 256) return false;
  if (P.N > 0x3fffffff) return false;
  return true;
}

int plan_halo(const Problem& P, bool pair, int sms, TcPlan& plan) {
  bool rank5 = false;
  if (!halo_fits(P, rank5)) return CONV_EUNSUPPORTED;
  TcArgs& a = plan.args;
  std::memset(&a, 0, sizeof(a));
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C; a.O = P.O;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.sd = P.s[0]; a.sh = P.s[1]; a.sw = P.s[2];
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.G = P.G; a.Cg = P.Cg; a.Og = P.Og;
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.M = P.M;
  a.K = static_cast<int>(P.K);
  a.BN = std::min(256, round_up(P.Og, 32));
  a.n_tiles = (P.Og + a.BN - 1) / a.BN;
  a.tile_h = kHaloTileH;
  a.tile_w = kHaloTileW;
  a.tiles_h = (P.Ho + (pair ? 2 : 1) * kHaloTileH - 1) / ((pair ? 2 : 1) * kHaloTileH);
  a.tiles_w = (P.Wo + kHaloTileW - 1) / kHaloTileW;
  const long long tt = static_cast<long long>(P.G) * P.N * P.Do * a.tiles_h * a.tiles_w * a.n_tiles;
  if (tt > 0x7fffffffLL) return CONV_EINVAL;
  a.total_tiles = static_cast<int>(tt);
  a.m_tiles = 0;
  a.kc = (P.Cg % 64 == 0) ? 64 : 32;
  a.cchunks = P.Cg / a.kc;
  a.kblocks = P.kD * P.kH * P.kW * a.cchunks;
  a.rank5 = rank5 ? 1 : 0;
  a.layout_type = a.kc == 64 ? 2u : 4u;    // 128-byte or 64-byte swizzle
  a.sbo = static_cast<uint32_t>(8 * a.kc * 2);  // one 8-row atom = one strip row of 8 pixels
  // one strip per (chunk, kd, kw): (16 + dh*(kH-1)) rows x 8 pixels x kc channels
  a.halo_w = kHaloTileW;
  a.halo_h = kHaloTileH + P.d[1] * (P.kH - 1);
  a.halo_bytes = static_cast<uint32_t>(a.halo_w * a.halo_h * a.kc * 2);
  a.halo_slot_bytes = (a.halo_bytes + 1023u) & ~1023u;
  a.a_bytes = 0;
  a.b_bytes = static_cast<uint32_t>((pair ? a.BN / 2 : a.BN) * a.kc * 2);
  a.sub_bytes = a.b_bytes;
  // the weight and strip rings are independent (a stage may span any number of
  // strip groups): first up to three weight stages beside two strip slots,
  // then as many more strip slots (up to 8) as the rest of shared memory holds
  // -- one strip serves only kH K blocks, so its load latency needs a deep ring
  const long long budget = static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(TcSmemTail)) - 64;
  int stages = 0;
  a.kbs = choose_kbs(a.BN, a.kc, a.b_bytes, budget - 2LL * a.halo_slot_bytes, 16, stages);
  if (stages < 2) return CONV_EUNSUPPORTED;
  stages = std::min(stages, 3);
  const long long left = budget - static_cast<long long>(stages) * a.kbs * a.b_bytes;
  a.a_slots = static_cast<int>(std::min<long long>(8, left / a.halo_slot_bytes));
  if (a.a_slots < 2) return CONV_EUNSUPPORTED;
  a.stages = stages;
  a.stage_bytes = static_cast<uint32_t>(a.kbs) * a.b_bytes;
  const uint32_t ab = P.dtype == CONV_BF16 ? 1u : 0u;
  const uint32_t mma_m = pair ? 2 * kBM : kBM;
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (static_cast<uint32_t>(a.BN >> 3) << 17) | ((mma_m >> 4) << 24);
  a.tmem_cols = next_pow2_cols(static_cast<uint32_t>(2 * a.BN));
  a.timeout_ns = kWaitTimeoutNs;
  plan.variant = pair ? CONV_VARIANT_TC_HALO_PAIR : CONV_VARIANT_TC_HALO;
  plan.pair = pair;
  plan.ctas = pair ? 2 * std::min(a.total_tiles, sms / 2) : std::min(a.total_tiles, sms);
  plan.smem = static_cast<size_t>(a.a_slots) * a.halo_slot_bytes + static_cast<size_t>(a.stages) * a.stage_bytes +
              1024 + sizeof(TcSmemTail) + 64;
  return CONV_OK;
}

// Transposed orientation: M = 128 output channels, N = BP output pixels.
// Needs what the im2col kernels need plus whole 128-channel tiles per group.
// BP = 256 when that still gives every SM a tile, else 128.
int plan_tc_t(const Problem& P, int sms, TcPlan& plan) {
  bool rank5 = false;
  if (!tma_fits(P, rank5) || P.Og % kTO != 0) return CONV_EUNSUPPORTED;
  if (P.M > 0x7fffffffLL - 256) return CONV_EUNSUPPORTED;  // TMA store row coordinate
  TcArgs& a = plan.args;
  std::memset(&a, 0, sizeof(a));
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C; a.O = P.O;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.sd = P.s[0]; a.sh = P.s[1]; a.sw = P.s[2];
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.G = P.G; a.Cg = P.Cg; a.Og = P.Og;
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.M = P.M;
  a.K = static_cast<int>(P.K);
  a.n_tiles = P.Og / kTO;
  const long long wide_tiles = (P.M + 255) / 256 * a.n_tiles * P.G;
  a.BN = wide_tiles >= sms ? 256 : 128;  // output pixels per tile (MMA N)
  const long long mt = (P.M + a.BN - 1) / a.BN;
  const long long tt = mt * a.n_tiles * P.G;
  if (tt > 0x7fffffffLL) return CONV_EINVAL;
  a.m_tiles = static_cast<int>(mt);
  a.total_tiles = static_cast<int>(tt);
  a.kc = (P.Cg % 64 == 0) ? 64 : (P.Cg % 32 == 0 ? 32 : 16);
  a.cchunks = P.Cg / a.kc;
  a.kblocks = P.kD * P.kH * P.kW * a.cchunks;
  a.rank5 = rank5 ? 1 : 0;
  a.layout_type = a.kc == 64 ? 2u : (a.kc == 32 ? 4u : 6u);
  a.sbo = static_cast<uint32_t>(8 * a.kc * 2);
  a.a_bytes = static_cast<uint32_t>(kTO * a.kc * 2);    // weight tile
  a.b_bytes = static_cast<uint32_t>(a.BN * a.kc * 2);   // patch rows
  a.sub_bytes = a.a_bytes + a.b_bytes;
  const long long avail = static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(TcSmemTail)) -
                          64 - 2LL * kTEpiGroups * kTEpiBytes;
  int stages = 0;
  a.kbs = choose_kbs(a.BN, a.kc, a.sub_bytes, avail, 8, stages);
  if (stages < 2) return CONV_EUNSUPPORTED;
  a.stages = stages;
  a.stage_bytes = static_cast<uint32_t>(a.kbs) * a.sub_bytes;
  const uint32_t ab = P.dtype == CONV_BF16 ? 1u : 0u;
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (static_cast<uint32_t>(a.BN >> 3) << 17) |
            ((static_cast<uint32_t>(kTO) >> 4) << 24);
  a.tmem_cols = next_pow2_cols(static_cast<uint32_t>(2 * a.BN));
  a.timeout_ns = kWaitTimeoutNs;
  plan.variant = CONV_VARIANT_TC_TMA_T;
  plan.pair = false;
  plan.ctas = std::min(a.total_tiles, sms);
  plan.smem = static_cast<size_t>(a.stages) * a.stage_bytes + 2 * kTEpiGroups * static_cast<size_t>(kTEpiBytes) +
              1024 + sizeof(TcSmemTail) + 64;
  return CONV_OK;
}

// Transposed orientation with halo reuse: M = 128 output channels, N = a
// tile_h x 8 block of output pixels read as views of one 8-pixel-wide input
// strip per (64-channel chunk, kd, kw).  Stride 1, C/G % 64 == 0,
// O/G % 128 == 0.  With `pair`, two CTAs issue M = 256 (128 output channels
// each) over the same block; each loads the strip of half the block's rows.
int plan_halo_t(const Problem& P, bool pair, int sms, TcPlan& plan) {
  // output channels per CTA: 128, or 64 when O/G is an odd multiple of 64
  // (an M = 64 instruction takes as long as M = 128 on B200, so 64 only when
  // 128 does not divide O/G); channel chunks of 64, or 32
  const int mo = (P.Og % kTO == 0 || pair) ? kTO : 64;
  const int o_tile = pair ? 2 * mo : mo;
  if (P.dtype == CONV_F32 || P.Cg % 32 != 0 || P.Og % o_tile != 0) return CONV_EUNSUPPORTED;
  if (P.s[0] != 1 || P.s[1] != 1 || P.s[2] != 1) return CONV_EUNSUPPORTED;
  if (P.N > 0x3fffffff) return CONV_EUNSUPPORTED;
  const bool rank5 = !is_2d(P);
  // block height: the multiple of 4 up to 32 that wastes the fewest rows of
  // Ho (ties to the taller block, which reuses the strip over more rows)
  int bh = kHTBlockHMax;
  {
    long long best = -1;
    for (int h = kHTBlockHMax; h >= 16; h -= 4) {
      const long long covered = static_cast<long long>((P.Ho + h - 1) / h) * h;
      if (best < 0 || covered < best) {
        best = covered;
        bh = h;
      }
    }
  }
  const long long hw = kHTBlockW;  // one strip per width tap
  const long long hh = (pair ? bh / 2 : bh) + static_cast<long long>(P.d[1]) * (P.kH - 1);  // rows per CTA
  if (hh > 256) return CONV_EUNSUPPORTED;
  TcArgs& a = plan.args;
  std::memset(&a, 0, sizeof(a));
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C; a.O = P.O;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.sd = P.s[0]; a.sh = P.s[1]; a.sw = P.s[2];
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.G = P.G; a.Cg = P.Cg; a.Og = P.Og;
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.M = P.M;
  a.K = static_cast<int>(P.K);
  a.BN = bh * kHTBlockW;  // MMA N: output pixels per tile
  a.n_tiles = P.Og / o_tile;
  a.tile_h = bh;
  a.tile_w = kHTBlockW;
  a.tiles_h = (P.Ho + bh - 1) / bh;
  a.tiles_w = (P.Wo + kHTBlockW - 1) / kHTBlockW;
  const long long tt = static_cast<long long>(P.G) * P.N * P.Do * a.tiles_h * a.tiles_w * a.n_tiles;
  if (tt > 0x7fffffffLL) return CONV_EINVAL;
  a.total_tiles = static_cast<int>(tt);
  a.m_tiles = 0;
  a.halo_w = static_cast<int>(hw);
  a.halo_h = static_cast<int>(hh);
  a.kc = (P.Cg % 64 == 0) ? 64 : 32;
  a.halo_bytes = static_cast<uint32_t>(hw * hh * a.kc * 2);
  a.halo_slot_bytes = (a.halo_bytes + 1023u) & ~1023u;
  // Resident weights: with one group and one output-channel tile every tile
  // multiplies by the same weights, so when they fit beside two strip slots
  // (with two epilogue staging tiles, else one) they are loaded once per CTA
  // instead of once per tile.
  const long long base_budget =
      static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(TcSmemTail)) - 64;
  const long long w_total = static_cast<long long>(P.kD) * P.kH * P.kW * P.Cg * mo * 2;
  a.w_resident = 0;
  a.epi_bufs = 2;
  if (P.G == 1 && a.n_tiles == 1) {
    for (int bufs = 2; bufs >= 1; --bufs) {
      if (base_budget - bufs * static_cast<long long>(kTEpiBytes) - w_total >= 2LL * a.halo_slot_bytes) {
        a.w_resident = 1;
        a.epi_bufs = bufs;
        break;
      }
    }
  }
  a.a_slots = 2;
  a.mo = mo;
  a.cchunks = P.Cg / a.kc;
  a.kblocks = P.kD * P.kH * P.kW * a.cchunks;
  a.rank5 = rank5 ? 1 : 0;
  a.layout_type = a.kc == 64 ? 2u : 4u;          // 128-byte or 64-byte swizzle
  a.sbo = static_cast<uint32_t>(8 * a.kc * 2);  // one atom = one strip row of 8 pixels
  a.a_bytes = 0;
  a.b_bytes = static_cast<uint32_t>(mo * a.kc * 2);  // one weight tile: mo channels x kc
  a.sub_bytes = a.b_bytes;
  // the weight and strip rings are independent: first up to three weight
  // stages beside two strip slots (or the one resident stage), then as many
  // more strip slots (up to 8) as the rest of shared memory holds
  const long long budget = base_budget - a.epi_bufs * static_cast<long long>(kTEpiBytes);
  int stages = 0;
  if (a.w_resident) {
    a.kbs = a.kblocks;
    stages = 1;
  } else {
    a.kbs = choose_kbs(a.BN, a.kc, a.b_bytes, budget - 2LL * a.halo_slot_bytes, 16, stages);
    if (stages < 2) return CONV_EUNSUPPORTED;
    stages = std::min(stages, 3);
  }
  const long long left = budget - static_cast<long long>(stages) * a.kbs * a.b_bytes;
  a.a_slots = static_cast<int>(std::min<long long>(8, left / a.halo_slot_bytes));
  if (a.a_slots < 2) return CONV_EUNSUPPORTED;
  a.stages = stages;
  a.stage_bytes = static_cast<uint32_t>(a.kbs) * a.b_bytes;
  const uint32_t ab = P.dtype == CONV_BF16 ? 1u : 0u;
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (static_cast<uint32_t>(a.BN >> 3) << 17) |
            ((static_cast<uint32_t>(o_tile) >> 4) << 24);
  a.tmem_cols = 2 * kHTAccStride;
  a.timeout_ns = kWaitTimeoutNs;
  plan.variant = pair ? CONV_VARIANT_TC_HALO_T_PAIR : CONV_VARIANT_TC_HALO_T;
  plan.pair = pair;
  plan.ctas = pair ? 2 * std::min(a.total_tiles, sms / 2) : std::min(a.total_tiles, sms);
  plan.smem = static_cast<size_t>(a.a_slots) * a.halo_slot_bytes + static_cast<size_t>(a.stages) * a.stage_bytes +
              static_cast<size_t>(a.epi_bufs) * kTEpiBytes + 1024 + sizeof(TcSmemTail) + 64;
  return CONV_OK;
}

// Phase-packed kernel (conv_phase.cuh) for 2-D layers with few input
// channels: one GEMM row = P output pixels of a row, P the smallest count
// whose windows start a multiple of 8 elements apart in the flattened input
// row; N = P*O <= 256; CTA pairs, each CTA ph_rows output rows of a tile.
int plan_phase(const Problem& P, int sms, TcPlan& plan) {
  if (P.dtype == CONV_F32 || P.G != 1) return CONV_EUNSUPPORTED;
  if (!is_2d(P)) return CONV_EUNSUPPORTED;
  if (P.d[2] != 1) return CONV_EUNSUPPORTED;  // a filter row's taps are contiguous
  const int sh = P.s[1], sw = P.s[2];
  if (P.H % sh != 0) return CONV_EUNSUPPORTED;  // input rows as (ih / sh, ih % sh)
  const long long WC = static_cast<long long>(P.W) * P.C;
  if ((WC * 2) % 16 != 0 || static_cast<long long>(P.N) * P.H * WC > 0x7fffffffLL) return CONV_EUNSUPPORTED;
  int Pg = 1;
  while ((Pg * sw * P.C) % 8 != 0) ++Pg;
  const int BN = Pg * P.O;
  // (the epilogue reads the accumulator 32 columns at a time)
  if (BN > 256 || BN % 32 != 0 || P.Wo % Pg != 0) return CONV_EUNSUPPORTED;
  const int qtot = P.Wo / Pg;
  const int al = round_up(P.p[2] * P.C, 8);
  const long long pitch = static_cast<long long>(Pg) * sw * P.C;
  const int span = al - P.p[2] * P.C + (Pg - 1) * sw * P.C + P.kW * P.C;
  const int Kw = round_up(span, 16);
  if (Kw > kPhWin) return CONV_EUNSUPPORTED;
  // windows are loaded kPhWin elements wide (128-byte rows); the MMAs read Kw
  int nleft = 0;
  while (nleft < qtot && pitch * nleft - al < 0) ++nleft;
  int nright = 0;
  while (nright < qtot - nleft && pitch * (qtot - 1 - nright) - al + kPhWin > WC) ++nright;
  const int qint = qtot - nleft - nright;
  const int nedge = nleft + nright;
  if (qint < 1 || qint > 256) return CONV_EUNSUPPORTED;
  int R = 0;
  for (int r = 8; r >= 1; r /= 2) {
    if (round_up(r * qint, 8) + 8 * nedge <= kBM) {
      R = r;
      break;
    }
  }
  if (R == 0) return CONV_EUNSUPPORTED;
  TcArgs& a = plan.args;
  std::memset(&a, 0, sizeof(a));
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C; a.O = P.O;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.sd = P.s[0]; a.sh = P.s[1]; a.sw = P.s[2];
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.G = P.G; a.Cg = P.Cg; a.Og = P.Og;
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.M = P.M;
  a.K = static_cast<int>(P.K);
  a.BN = BN;
  a.ph_P = Pg;
  a.ph_ks = Kw / 16;
  a.ph_qtot = qtot;
  a.ph_qint = qint;
  a.ph_nleft = nleft;
  a.ph_nright = nright;
  a.ph_rows = R;
  a.ph_erow0 = round_up(R * qint, 8);
  a.ph_align = al;
  a.ph_wbytes = static_cast<uint32_t>(P.w_bytes);
  a.ph_bblk = static_cast<uint32_t>(BN / 2 * 128);  // per CTA: BN/2 rows of 128 bytes
  a.ph_gcols = BN % 64 == 0 ? 64 : 32;  // store rows of 128 (or 64) bytes
  // the two staging tiles also hold the copy of w that B is built from
  a.ph_epi_bytes = static_cast<uint32_t>(
      std::max<long long>(round_up(R * qtot * 2 * a.ph_gcols, 1024), (static_cast<long long>(P.w_bytes) / 2 + 1023) / 1024 * 1024));
  a.tiles_h = (P.Ho + 2 * R - 1) / (2 * R);  // a pair tile: 2 * ph_rows output rows
  const long long tt = static_cast<long long>(P.N) * a.tiles_h;
  if (tt > 0x7fffffffLL) return CONV_EINVAL;
  a.total_tiles = static_cast<int>(tt);
  a.stage_bytes = kPhAStage;
  const long long b_bytes = static_cast<long long>(P.kH) * a.ph_bblk;
  const long long avail = static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(TcSmemTail)) -
                          64 - b_bytes - 2LL * a.ph_epi_bytes;
  if (avail < 2LL * a.stage_bytes) return CONV_EUNSUPPORTED;
  a.stages = static_cast<int>(std::min<long long>(6, avail / a.stage_bytes));
  if (static_cast<long long>(P.w_bytes) > 2LL * a.ph_epi_bytes) return CONV_EUNSUPPORTED;
  const uint32_t ab = P.dtype == CONV_BF16 ? 1u : 0u;
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
            ((static_cast<uint32_t>(2 * kBM) >> 4) << 24);
  a.tmem_cols = next_pow2_cols(static_cast<uint32_t>(2 * BN));
  a.timeout_ns = kWaitTimeoutNs;
  plan.variant = CONV_VARIANT_TC_PHASE;
  plan.pair = true;
  plan.ctas = 2 * std::min(a.total_tiles, sms / 2);
  plan.smem = static_cast<size_t>(a.stages) * a.stage_bytes + static_cast<size_t>(b_bytes) +
              2 * static_cast<size_t>(a.ph_epi_bytes) + 1024 + sizeof(TcSmemTail) + 64;
  return CONV_OK;
}

// Sub-pixel phases of a transposed convolution on the gather kernel: output
// pixel q (per dimension) is reached only by taps k with
// (q - p_lo + k*d) divisible by the input dilation s, and that set depends on
// q mod s alone.  Each phase gets its own m tiles and reads only its taps, so
// no MMA multiplies an inserted zero.  Needs 64-channel K blocks (Cg % 64 ==
// 0, one tap per K block) and at most kMaxTp non-empty phases.
bool plan_tp(const Problem& P, TcArgs& a) {
  if (!P.wtrans || a.gather_mode != GATHER_VEC8 || P.Cg % 64 != 0) return false;
  if (P.idil[0] == 1 && P.idil[1] == 1 && P.idil[2] == 1) return false;
  const int k[3] = {P.kD, P.kH, P.kW};
  const int Q[3] = {P.Do, P.Ho, P.Wo};
  int A[3][64], k0[3][64], nk[3][64], c0[3][64];
  for (int i = 0; i < 3; ++i) {
    const int sd = P.idil[i];
    if (sd > 64) return false;
    int g = sd, b = P.d[i];
    while (b) { const int t = g % b; g = b; b = t; }  // gcd(s, d)
    a.tp_step[i] = sd / g;
    a.tp_dstep[i] = P.d[i] / g;
    for (int r = 0; r < sd; ++r) {
      A[i][r] = r < Q[i] ? (Q[i] - r + sd - 1) / sd : 0;
      k0[i][r] = 0;
      nk[i][r] = 0;
      c0[i][r] = 0;
      for (int kk = 0; kk < k[i]; ++kk) {
        const long long v = static_cast<long long>(r) - P.p[i] + static_cast<long long>(kk) * P.d[i];
        if (((v % sd) + sd) % sd == 0) {
          if (nk[i][r] == 0) {
            k0[i][r] = kk;
            c0[i][r] = static_cast<int>(v / sd);  // exact
          }
          ++nk[i][r];
        }
      }
    }
  }
  int count = 0;
  long long tiles = 0;
  for (int rd = 0; rd < P.idil[0]; ++rd)
    for (int rh = 0; rh < P.idil[1]; ++rh)
      for (int rw = 0; rw < P.idil[2]; ++rw) {
        const long long Mph = static_cast<long long>(P.N) * A[0][rd] * A[1][rh] * A[2][rw];
        if (Mph == 0) continue;
        if (count == kMaxTp || Mph > 0x7fffffffLL - kBM) return false;
        const int rr[3] = {rd, rh, rw};
        for (int i = 0; i < 3; ++i) {
          a.tp_r[count][i] = rr[i];
          a.tp_A[count][i] = A[i][rr[i]];
          a.tp_k0[count][i] = k0[i][rr[i]];
          a.tp_nk[count][i] = nk[i][rr[i]];
          a.tp_c0[count][i] = c0[i][rr[i]];
        }
        a.tp_tbase[count] = static_cast<int>(tiles);
        tiles += (Mph + kBM - 1) / kBM;
        if (tiles > 0x7fffffffLL) return false;
        ++count;
      }
  a.tp_tbase[count] = static_cast<int>(tiles);
  a.tp_count = count;
  a.tp_cpt = P.Cg / 64;
  a.m_tiles = static_cast<int>(tiles);
  const long long tt = tiles * a.n_tiles * P.G;
  if (tt > 0x7fffffffLL) return false;
  a.total_tiles = static_cast<int>(tt);
  a.tp_on = 1;
  return true;
}

int plan_tc(const Problem& P, int variant, int sms, TcPlan& plan) {
  // input dilation and transposed weights: the gather kernel only
  if (!plain_input(P) && variant != CONV_VARIANT_TC_GATHER) return CONV_EUNSUPPORTED;
  if (variant == CONV_VARIANT_TC_PHASE) return plan_phase(P, sms, plan);
  if (variant == CONV_VARIANT_TC_HALO_T || variant == CONV_VARIANT_TC_HALO_T_PAIR)
    return plan_halo_t(P, variant == CONV_VARIANT_TC_HALO_T_PAIR, sms, plan);
  if (variant == CONV_VARIANT_TC_HALO || variant == CONV_VARIANT_TC_HALO_PAIR)
    return plan_halo(P, variant == CONV_VARIANT_TC_HALO_PAIR, sms, plan);
  if (variant == CONV_VARIANT_TC_TMA_T) return plan_tc_t(P, sms, plan);
  if (P.dtype == CONV_F32) return CONV_EUNSUPPORTED;
  TcArgs& a = plan.args;
  std::memset(&a, 0, sizeof(a));
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C; a.O = P.O;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.sd = P.s[0]; a.sh = P.s[1]; a.sw = P.s[2];
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.G = P.G; a.Cg = P.Cg; a.Og = P.Og;
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.M = P.M;
  a.K = static_cast<int>(P.K);
  a.BN = std::min(256, round_up(P.Og, 32));
  a.n_tiles = (P.Og + a.BN - 1) / a.BN;
  // CTA pairs (256-row tiles) for the TMA path once there are enough tiles to
  // keep every SM pair busy; single CTAs (128-row tiles) otherwise.
  plan.pair = variant == CONV_VARIANT_TC_TMA_PAIR;
  const long long mt = plan.pair ? (P.M + 2 * kBM - 1) / (2 * kBM) : (P.M + kBM - 1) / kBM;
  const long long tt = mt * a.n_tiles * P.G;
  if (tt > 0x7fffffffLL) return CONV_EINVAL;
  a.m_tiles = static_cast<int>(mt);
  a.total_tiles = static_cast<int>(tt);
  bool rank5 = false;
  if (variant == CONV_VARIANT_TC_TMA || variant == CONV_VARIANT_TC_TMA_PAIR) {
    if (!tma_fits(P, rank5)) return CONV_EUNSUPPORTED;
    a.kc = (P.Cg % 64 == 0) ? 64 : (P.Cg % 32 == 0 ? 32 : 16);
    a.cchunks = P.Cg / a.kc;
    a.kblocks = P.kD * P.kH * P.kW * a.cchunks;
    a.rank5 = rank5 ? 1 : 0;
  } else {
    a.kc = 64;
    a.cchunks = 0;
    a.rank5 = 0;
    // gather layout of K: natural weight order (kd, kh, kw, c), except in span
    // layout where each filter row (kd, kh) is padded to Lp = roundup(kW*C, 8)
    if (P.Cg % 8 == 0) {
      a.gather_mode = GATHER_VEC8;
    } else if (P.G == 1 && P.d[2] == 1 && !P.flip && plain_input(P)) {  // (span layout: the filter's own tap order)
      a.gather_mode = GATHER_SPAN;
    } else {
      a.gather_mode = GATHER_SCALAR;
    }
    a.Lp = round_up(P.kW * P.C, 8);
    // Row staging: 2-D problems in span layout whose input rows are 16-byte
    // strided and whose 128-pixel tiles touch at most two images get their
    // input rows by TMA instead of per-thread loads.
    if (a.gather_mode == GATHER_SPAN && is_2d(P) &&
        (static_cast<long long>(P.W) * P.C) % 8 == 0 && static_cast<long long>(P.Ho) * P.Wo >= kBM) {
      // a row of row_e = W*C elements is one box row of n_boxes x box_e, with
      // box_e the largest multiple-of-8 divisor of row_e that is <= 256
      const long long we = static_cast<long long>(P.W) * P.C;
      int box_e = 0;
      for (int b = 256; b >= 32; b -= 8)
        if (we % b == 0) {
          box_e = b;
          break;
        }
      const long long n_boxes = box_e ? we / box_e : 0;
      const int orows = std::min(P.Ho, (kBM - 1) / P.Wo + 2);
      const long long stage_rows = static_cast<long long>(orows - 1) * P.s[1] + static_cast<long long>(P.kH - 1) * P.d[1] + 1;
      const long long seg = (stage_rows * we * 2 + 127) / 128 * 128;
      const long long rows_bytes = (2 * seg + 1023) / 1024 * 1024;
      if (box_e && n_boxes <= 256 && stage_rows <= 256 && 3 * rows_bytes <= 108 * 1024 &&
          P.N * static_cast<long long>(P.H) < (1LL << 31)) {
        a.gather_mode = GATHER_ROWS;
        a.box_e = box_e;
        a.n_boxes = static_cast<int>(n_boxes);
        a.stage_rows = static_cast<int>(stage_rows);
        a.row_e = static_cast<int>(we);
        a.seg_bytes = static_cast<uint32_t>(seg);
        a.rows_bytes = static_cast<uint32_t>(rows_bytes);
      }
    }
    const long long kp = (a.gather_mode == GATHER_SPAN || a.gather_mode == GATHER_ROWS)
                             ? static_cast<long long>(P.kD) * P.kH * a.Lp : P.K;
    if (kp > 0x7fffffffLL - 64) return CONV_EINVAL;
    a.Kp = static_cast<int>(kp);
    a.kblocks = static_cast<int>((kp + 63) / 64);
  }
  if (variant == CONV_VARIANT_TC_GATHER) plan_tp(P, a);
  a.x_elems = static_cast<long long>(P.x_bytes / P.esize);
  a.idil_on = plain_input(P) ? 0 : 1;
  a.idd = P.idil[0]; a.idh = P.idil[1]; a.idw = P.idil[2];
  a.wtrans = P.wtrans;
  a.layout_type = a.kc == 64 ? 2u : (a.kc == 32 ? 4u : 6u);
  a.sbo = static_cast<uint32_t>(8 * a.kc * 2);
  a.a_bytes = static_cast<uint32_t>(kBM * a.kc * 2);
  a.b_bytes = static_cast<uint32_t>((plan.pair ? a.BN / 2 : a.BN) * a.kc * 2);  // per CTA
  a.b_resident = 0;
  a.bres_bytes = 0;
  if (variant == CONV_VARIANT_TC_GATHER) {
    const long long bres = static_cast<long long>(a.kblocks) * a.BN * 128;
    if (P.G == 1 && a.n_tiles == 1 && bres <= kMaxResidentB) {
      a.b_resident = 1;
      a.bres_bytes = static_cast<uint32_t>(bres);
    }
  }
  a.sub_bytes = a.a_bytes + (a.b_resident ? 0u : a.b_bytes);
  // TMA-store epilogue: y rows 16-byte strided, every 32-channel box inside one
  // group (or clipped by the tensor's own extent when there is one group), row
  // coordinates within int32; the transposed-convolution phase tiles (rows not
  // consecutive) keep register stores
  a.y_tma = (P.O % 8 == 0 && (P.G == 1 || P.Og % 32 == 0) && P.M <= 0x7fffffffLL - 256 && !a.tp_on) ? 1 : 0;
  a.epi_bytes = a.y_tma ? kEpiRowBytes + 1024u : 0u;  // the staging buffers start on a 1 KB boundary
  const long long avail = static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(TcSmemTail)) - 64 -
                          a.bres_bytes - 3LL * a.rows_bytes - a.epi_bytes;
  int stages = 0;
  a.kbs = choose_kbs(a.BN, a.kc, a.sub_bytes, avail, 8, stages);
  if (stages < 2) return CONV_EUNSUPPORTED;
  a.stages = stages;
  a.stage_bytes = static_cast<uint32_t>(a.kbs) * a.sub_bytes;
  const uint32_t ab = P.dtype == CONV_BF16 ? 1u : 0u;
  const uint32_t mma_m = plan.pair ? 2 * kBM : kBM;
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (static_cast<uint32_t>(a.BN >> 3) << 17) |
            ((mma_m >> 4) << 24);
  a.tmem_cols = next_pow2_cols(static_cast<uint32_t>(2 * a.BN));
  a.timeout_ns = kWaitTimeoutNs;
  plan.variant = variant;
  plan.ctas = plan.pair ? 2 * std::min(a.total_tiles, sms / 2) : std::min(a.total_tiles, sms);
  plan.smem = static_cast<size_t>(a.stages) * a.stage_bytes + a.bres_bytes + 3 * static_cast<size_t>(a.rows_bytes) +
              a.epi_bytes + 1024 + sizeof(TcSmemTail) + 64;
  return CONV_OK;
}

// f32 -> SIMT.  f16/bf16 -> TMA im2col when it can describe the problem,
// else the in-kernel gather.  When the output channels per group come in
// 64- or 128-wide tiles that a 256-wide one cannot cover (O/G = 64, 128, 192,
// 384, ...): the transposed halo kernel at stride 1 with 32- or 64-channel
// chunks and kH >= 2 (each input strip then serves kH taps) and a tile for
// every SM, else (O/G a multiple of 128) the transposed im2col kernel when
// there are enough 256-pixel tiles for every SM.  Otherwise CTA pairs once there are at least as many 256-row tiles as
// SM pairs, else single CTAs.  Every choice here is the fastest measured on
// B200 for the shapes of the workload set; TC_HALO, TC_HALO_PAIR and
// TC_HALO_T_PAIR stay explicit (slower there than the choice made here).
// Depthwise kernels (conv_dw.cuh): one filter per channel (groups = C = O)
// with 16-byte channel vectors, P = 4 output pixels per thread.  The
// TMA-staged form (persistent CTAs, input slabs through an mbarrier ring) is
// the DEPTHWISE variant wherever its slabs fit; the direct form (loads from
// global memory, one block per CB x PB pixel groups) is DEPTHWISE_DIRECT and
// the fallback.
constexpr int kDwP = 4;
constexpr size_t kDwTmaSmem = 220 * 1024;

int dw_vec(const Problem& P) { return P.dtype == CONV_F32 ? 4 : 8; }

bool dw_fits(const Problem& P) {
  const long long taps = static_cast<long long>(P.kD) * P.kH * P.kW;
  return P.Cg == 1 && P.Og == 1 && (static_cast<long long>(P.C) * static_cast<long long>(P.esize)) % 16 == 0 &&
         taps * dw_vec(P) * 4 <= kDwSmemLimit && plain_input(P);
}

void dw_geometry(const Problem& P, DwArgs& a) {
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.sd = P.s[0]; a.sh = P.s[1]; a.sw = P.s[2];
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.wg = (P.Wo + kDwP - 1) / kDwP;
  a.flip = P.flip;
}

int plan_dw(const Problem& P, DwArgs& a, dim3& grid, dim3& block, size_t& smem) {
  if (!dw_fits(P)) return CONV_EUNSUPPORTED;
  dw_geometry(P, a);
  const int V = dw_vec(P);
  const int cvs = P.C / V;
  const long long taps = static_cast<long long>(P.kD) * P.kH * P.kW;
  int cb = std::min(cvs, kDwMaxCB);
  while (cb > 1 && taps * cb * V * 4 > kDwSmemLimit) cb = (cb + 1) / 2;
  a.cb = cb;
  a.pb = std::max(1, kDwThreads / cb);
  long long groups;
  if (!mul_ok(static_cast<long long>(P.N) * P.Do, static_cast<long long>(P.Ho) * a.wg, groups))
    return CONV_EINVAL;
  if (groups > 0x7fffffffLL - kDwThreads) return CONV_EUNSUPPORTED;
  a.groups = static_cast<int>(groups);
  const long long bx = (groups + a.pb - 1) / a.pb;
  const long long by = (cvs + cb - 1) / cb;
  if (bx > 0x7fffffffLL || by > 65535) return CONV_EUNSUPPORTED;
  grid = dim3(static_cast<unsigned>(bx), static_cast<unsigned>(by), 1);
  block = dim3(static_cast<unsigned>(cb * a.pb), 1, 1);
  smem = static_cast<size_t>(taps * cb * V) * sizeof(float);
  return CONV_OK;
}

// Consumer form of the TMA-staged kernel (the shapes measured fastest on
// B200 with each): 3x3 filters at equal strides 1 or 2 without dilation keep
// all nine weights in registers (16-bit types: four-row blocks at stride 1,
// two at stride 2, eight consumer warps; f32: two / one rows, twelve warps);
// 5- or 7-wide filters at width stride 1 or 2 without width dilation stream
// filter rows; anything else runs the generic consumer.
struct DwForm {
  int mode, K, S, R, ncw;
};

DwForm dw_tma_form(const Problem& P) {
  const bool w_plain = P.d[2] == 1 && (P.s[2] == 1 || P.s[2] == 2);
  if (P.kH == 3 && P.kW == 3 && P.s[1] == P.s[2] && P.d[1] == 1 && w_plain) {
    const bool s1 = P.s[1] == 1;
    if (P.esize == 2) return {kDwSquare, 3, P.s[1], s1 ? 4 : 2, 8};
    return {kDwSquare, 3, P.s[1], s1 ? 2 : 1, 12};
  }
  if ((P.kW == 5 || P.kW == 7) && w_plain) return {kDwRows, P.kW, P.s[2], 1, 8};
  return {kDwGeneric, 0, 0, 1, 8};
}

// Tile of the TMA-staged form: the consumer threads are cb channel vectors x
// BR x BC blocks of R x 4 output pixels (BC = 4 blocks across, BR to fill the
// consumer threads, no more rows than the output has); block rows, then columns,
// halved until the slab box fits TMA's 256-element box limit and two slabs
// fit beside the filters in `budget` bytes.
int dw_tma_tile(const Problem& P, DwTmaArgs& t, int R, int consumers, long long budget) {
  DwArgs& a = t.d;
  const long long VB = 4LL * P.esize;
  const long long taps = static_cast<long long>(P.kD) * P.kH * P.kW;
  const long long wbytes = (taps * a.cb * 16 + 15) / 16 * 16;
  const long long tail = static_cast<long long>(sizeof(DwTmaTail));
  const int nb = consumers / a.cb;
  t.BC = std::max(1, std::min({4, nb, (P.Wo + kDwTmaP - 1) / kDwTmaP}));
  t.BR = std::max(1, std::min(nb / t.BC, (P.Ho + R - 1) / R));
  while (true) {
    t.TH = t.BR * R;
    t.TW = t.BC * kDwTmaP;
    t.span_h = (t.TH - 1) * P.s[1] + (P.kH - 1) * P.d[1] + 1;
    t.span_w = (t.TW - 1) * P.s[2] + (P.kW - 1) * P.d[2] + 1;
    const long long slab = static_cast<long long>(t.span_h) * t.span_w * a.cb * VB;
    const long long pitch = (slab + 127) / 128 * 128;
    const long long room = budget - wbytes - tail;
    t.stages = room > 0 ? static_cast<int>(std::min<long long>(kDwTmaMaxStages, room / pitch)) : 0;
    if (t.span_h <= 256 && t.span_w <= 256 && t.stages >= 2) {
      t.slab_bytes = static_cast<uint32_t>(slab);
      t.slab_pitch = static_cast<uint32_t>(pitch);
      t.w_off = static_cast<uint32_t>(pitch * t.stages);
      t.tail_off = static_cast<uint32_t>(t.w_off + wbytes);
      return CONV_OK;
    }
    if (t.BR > 1) t.BR = (t.BR + 1) / 2;
    else if (t.BC > 1) t.BC = (t.BC + 1) / 2;
    else return CONV_EUNSUPPORTED;
  }
}

// Two CTAs share an SM (half the shared memory each) when the form's
// registers allow it and that leaves them two slabs or more; otherwise one CTA
// takes it all.  A specialised form falls back to the generic consumer if its
// tile does not fit.
int plan_dw_tma(const Problem& P, int sms, DwTmaArgs& t, DwForm& f, int& grid, size_t& smem) {
  if (!dw_fits(P)) return CONV_EUNSUPPORTED;
  std::memset(&t, 0, sizeof(t));
  DwArgs& a = t.d;
  dw_geometry(P, a);
  const int cvs = P.C / 4;  // channel vectors of 4
  t.nct = (cvs + 31) / 32;
  a.cb = (cvs + t.nct - 1) / t.nct;
  if (P.esize == 2) a.cb = (a.cb + 1) / 2 * 2;  // 16-byte aligned channel tiles (TMA x coordinate)
  if ((a.cb * 4 * P.esize) % 16 != 0 || a.cb > 32) return CONV_EUNSUPPORTED;
  f = dw_tma_form(P);
  int per_sm = 2;
  bool fit = false;
  for (int attempt = 0; attempt < 2 && !fit; ++attempt) {
    if (attempt == 1) {
      if (f.mode == kDwGeneric) break;
      f = {kDwGeneric, 0, 0, 1, 8};
    }
    per_sm = dw_tma_ctas_per_sm(f.mode, f.R, f.ncw);
    const int consumers = 32 * f.ncw;
    if (per_sm == 2 && dw_tma_tile(P, t, f.R, consumers, static_cast<long long>(kDwTmaSmem) / 2) == CONV_OK) {
      fit = true;
    } else if (dw_tma_tile(P, t, f.R, consumers, static_cast<long long>(kDwTmaSmem)) == CONV_OK) {
      per_sm = 1;
      fit = true;
    }
  }
  if (!fit) return CONV_EUNSUPPORTED;
  t.tiles_h = (P.Ho + t.TH - 1) / t.TH;
  t.tiles_w = (P.Wo + t.TW - 1) / t.TW;
  long long tiles;
  if (!mul_ok(static_cast<long long>(P.N) * P.Do, static_cast<long long>(t.tiles_h) * t.tiles_w, tiles))
    return CONV_EINVAL;
  if (tiles > 0x7fffffffLL) return CONV_EUNSUPPORTED;
  t.tiles = static_cast<int>(tiles);
  const long long per_ct =
      std::max<long long>(1, std::min<long long>(static_cast<long long>(sms) * per_sm / t.nct, tiles));
  const long long g = per_ct * t.nct;
  if (g > 0x7fffffffLL) return CONV_EUNSUPPORTED;
  grid = static_cast<int>(g);
  smem = t.tail_off + sizeof(DwTmaTail);
  t.timeout_ns = kWaitTimeoutNs;
  return CONV_OK;
}

// x as a 5-D tensor (C, W, H, D, N); box = one slab of a channel tile.
int encode_dw_map(const Problem& P, const DwTmaArgs& t, const void* x, CUtensorMap& m) {
  std::memset(&m, 0, sizeof(m));
  const DriverFns& drv = driver_fns();
  if (!drv.tiled) return CONV_EDRIVER;
  const CUtensorMapDataType dt = P.dtype == CONV_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t e = static_cast<cuuint64_t>(P.esize);
  const cuuint64_t C = P.C, W = P.W, H = P.H, D = P.D;
  cuuint64_t dim[5] = {C, W, H, D, static_cast<cuuint64_t>(P.N)};
  cuuint64_t str[4] = {e * C, e * C * W, e * C * W * H, e * C * W * H * D};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(t.d.cb * 4), static_cast<cuuint32_t>(t.span_w),
                       static_cast<cuuint32_t>(t.span_h), 1u, 1u};
  cuuint32_t est[5] = {1, 1, 1, 1, 1};
  const CUresult r = drv.tiled(&m, dt, 5, const_cast<void*>(x), dim, str, box, est, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(m, P.x_bytes, drv.driver_version);
  return CONV_OK;
}

// Raises a kernel's dynamic shared-memory limit to the 227 KB maximum once
// per device (bit `dev` of `done`; devices beyond 63 set it every launch).
template <typename Kern>
cudaError_t dw_smem_attr(Kern* k, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 63;
  const uint64_t bit = dev < 63 ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

template <typename T, int V, int KW, int SW, int DW>
cudaError_t launch_dw_t(const DwArgs& a, dim3 grid, dim3 block, size_t smem, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  auto* k = conv_fwd_dw_direct_kernel<T, V, kDwP, KW, SW, DW>;
  if (smem > 48 * 1024) {
    const cudaError_t e = dw_smem_attr(k, attr_done);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(k, grid, block, smem, st, 1, a);
}

template <typename T, int MODE, int K, int S, int R, int NCW>
cudaError_t launch_dw_tma_t(const CUtensorMap& m, const DwTmaArgs& t, int grid, size_t smem, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  auto* k = conv_fwd_dw_tma_kernel<T, MODE, K, S, R, NCW>;
  const cudaError_t e = dw_smem_attr(k, attr_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), dim3(32 * (NCW + 1)), smem, st, 1, m, t);
}

// The filter-row forms compiled with their width, stride and dilation fixed
// (the register window); any other width runs the generic form.
template <typename T, int V>
cudaError_t launch_dw_shape(const DwArgs& a, dim3 grid, dim3 block, size_t smem, cudaStream_t st) {
  if (a.dw == 1 && a.sw == 1) {
    if (a.kW == 3) return launch_dw_t<T, V, 3, 1, 1>(a, grid, block, smem, st);
    if (a.kW == 5) return launch_dw_t<T, V, 5, 1, 1>(a, grid, block, smem, st);
    if (a.kW == 7) return launch_dw_t<T, V, 7, 1, 1>(a, grid, block, smem, st);
  }
  if (a.dw == 1 && a.sw == 2 && a.kW == 3) return launch_dw_t<T, V, 3, 2, 1>(a, grid, block, smem, st);
  return launch_dw_t<T, V, 0, 0, 0>(a, grid, block, smem, st);
}

// One instantiation per form dw_tma_form returns (16-bit and f32 square
// forms differ in rows and warps).
template <typename T>
cudaError_t launch_dw_tma_form(const CUtensorMap& m, const DwTmaArgs& t, const DwForm& f, int grid, size_t smem,
                               cudaStream_t st) {
  constexpr bool h = sizeof(T) == 2;
  if (f.mode == kDwSquare && f.S == 1)
    return launch_dw_tma_t<T, kDwSquare, 3, 1, h ? 4 : 2, h ? 8 : 12>(m, t, grid, smem, st);
  if (f.mode == kDwSquare && f.S == 2)
    return launch_dw_tma_t<T, kDwSquare, 3, 2, h ? 2 : 1, h ? 8 : 12>(m, t, grid, smem, st);
  if (f.mode == kDwRows) {
    if (f.K == 5 && f.S == 1) return launch_dw_tma_t<T, kDwRows, 5, 1, 1, 8>(m, t, grid, smem, st);
    if (f.K == 5 && f.S == 2) return launch_dw_tma_t<T, kDwRows, 5, 2, 1, 8>(m, t, grid, smem, st);
    if (f.K == 7 && f.S == 1) return launch_dw_tma_t<T, kDwRows, 7, 1, 1, 8>(m, t, grid, smem, st);
    if (f.K == 7 && f.S == 2) return launch_dw_tma_t<T, kDwRows, 7, 2, 1, 8>(m, t, grid, smem, st);
  }
  return launch_dw_tma_t<T, kDwGeneric, 0, 0, 1, 8>(m, t, grid, smem, st);
}

int launch_dw_direct(const Problem& P, const void* x, const void* w, void* y, cudaStream_t st) {
  DwArgs a;
  dim3 grid, block;
  size_t smem;
  const int rc = plan_dw(P, a, grid, block, smem);
  if (rc != CONV_OK) return rc;
  a.x = x; a.w = w; a.y = y;
  cudaError_t e;
  if (P.dtype == CONV_F32) e = launch_dw_shape<float, 4>(a, grid, block, smem, st);
  else if (P.dtype == CONV_F16) e = launch_dw_shape<__half, 8>(a, grid, block, smem, st);
  else e = launch_dw_shape<__nv_bfloat16, 8>(a, grid, block, smem, st);
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

int launch_dw(const Problem& P, const void* x, const void* w, void* y, cudaStream_t st, int sms) {
  DwTmaArgs t;
  DwForm f;
  int grid;
  size_t smem;
  if (plan_dw_tma(P, sms, t, f, grid, smem) != CONV_OK) return launch_dw_direct(P, x, w, y, st);
  t.d.x = x; t.d.w = w; t.d.y = y;
  t.inject_stall = 0;
  const unsigned long long stall_ns = g_inject_stall_ns.exchange(0);
  if (stall_ns != 0) {
    t.inject_stall = 1;
    t.timeout_ns = stall_ns;
  }
  CUtensorMap m;
  const int rc = encode_dw_map(P, t, x, m);
  if (rc != CONV_OK) return rc;
  cudaError_t e;
  if (P.dtype == CONV_F32) e = launch_dw_tma_form<float>(m, t, f, grid, smem, st);
  else if (P.dtype == CONV_F16) e = launch_dw_tma_form<__half>(m, t, f, grid, smem, st);
  else e = launch_dw_tma_form<__nv_bfloat16>(m, t, f, grid, smem, st);
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

// ---------------------------------------------------------------- transposed convolution by phases

// The phase decomposition of a transposed convolution (conv_tconv.cuh) and
// whether the TMA-fed phase kernel can run it.  The Problem of a transposed
// convolution holds the undilated input extents, the stride as input dilation
// (idil), padding p_lo = d(k-1) - pad and p_hi = p_lo + out_pad.
int plan_tconv(const Problem& P, int sms, TconvArgs& a, int& ctas, size_t& smem) {
  if (!P.wtrans || (P.dtype != CONV_F16 && P.dtype != CONV_BF16)) return CONV_EUNSUPPORTED;
  if (P.Cg % 64 != 0 || P.Og % 128 != 0 || P.O % 8 != 0) return CONV_EUNSUPPORTED;
  std::memset(&a, 0, sizeof(a));
  const int in[3] = {P.D, P.H, P.W}, k[3] = {P.kD, P.kH, P.kW}, out[3] = {P.Do, P.Ho, P.Wo};
  int maxoff[3];
  for (int i = 0; i < 3; ++i) {
    const int s = P.idil[i];
    if (P.d[i] != 1 || s > kTcvMaxStride) return CONV_EUNSUPPORTED;
    const int pad = (k[i] - 1) - P.p[i];
    a.s[i] = s;
    int lower = 0, moff = 0, tm = 0;
    bool any = false;
    for (int r = 0; r < s; ++r) {
      const int kr = (r + pad) % s;
      const int J = kr < k[i] ? (k[i] - kr + s - 1) / s : 0;
      const int c = (r + pad - kr) / s;
      const int T = out[i] > r ? (out[i] - r + s - 1) / s : 0;
      a.ph_k[i][r] = kr;
      a.ph_J[i][r] = J;
      a.ph_c[i][r] = c;
      a.ph_T[i][r] = T;
      tm = std::max(tm, T);
      if (J > 0) {
        lower = any ? std::min(lower, c - J + 1) : c - J + 1;
        moff = any ? std::max(moff, c) : c;
        any = true;
      }
    }
    a.lower[i] = lower;
    a.Tm[i] = tm;
    maxoff[i] = moff - lower;
  }
  // 2-D problems (one input plane, one filter plane) use a rank-4 walk
  const bool rank5 = !(P.D == 1 && P.kD == 1 && P.Do == 1 && a.s[0] == 1 && a.lower[0] == 0);
  const int lo = rank5 ? -16 : -128, hi = rank5 ? 15 : 127;
  for (int i = rank5 ? 0 : 1; i < 3; ++i) {
    const long long upper = static_cast<long long>(a.Tm[i]) - in[i] + a.lower[i];
    if (a.lower[i] < lo || a.lower[i] > hi || upper < lo || upper > hi || maxoff[i] > hi) return CONV_EUNSUPPORTED;
  }
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.Cin = P.C; a.Cout = P.O;
  a.G = P.G; a.Cig = P.Cg; a.Cog = P.Og;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.Qd = P.Do; a.Qh = P.Ho; a.Qw = P.Wo;
  a.rank5 = rank5 ? 1 : 0;
  a.Mph = static_cast<long long>(P.N) * a.Tm[0] * a.Tm[1] * a.Tm[2];
  if (a.Mph > 0x7fffffffLL - 512) return CONV_EUNSUPPORTED;
  a.nphase = a.s[0] * a.s[1] * a.s[2];
  a.BN = P.Og % 256 == 0 ? 256 : 128;
  a.n_tiles = P.Og / a.BN;
  a.m_tiles = static_cast<int>((a.Mph + 255) / 256);
  const long long tt = static_cast<long long>(a.nphase) * P.G * a.n_tiles * a.m_tiles;
  if (tt > 0x7fffffffLL) return CONV_EUNSUPPORTED;
  a.total_tiles = static_cast<int>(tt);
  // 128 input channels per sub-block where possible: 16 KB TMA boxes (half the
  // operations per byte of 64-channel ones)
  a.kc = P.Cg % 128 == 0 ? 128 : 64;
  a.cchunks = P.Cg / a.kc;
  a.a_bytes = static_cast<uint32_t>(kBM * a.kc * 2);                   // 128 pixels x kc channels
  a.b_bytes = static_cast<uint32_t>((a.BN / 2 / 64) * a.kc * 128);     // this CTA's [kc][64] weight boxes
  a.sub_bytes = a.a_bytes + a.b_bytes;
  const long long avail = static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(TcSmemTail)) - 64;
  int stages = 0;
  a.kbs = choose_kbs(a.BN, a.kc, a.sub_bytes, avail, 8, stages);
  if (stages < 2) return CONV_EUNSUPPORTED;
  a.stages = stages;
  a.stage_bytes = static_cast<uint32_t>(a.kbs) * a.sub_bytes;
  const uint32_t ab = P.dtype == CONV_BF16 ? 1u : 0u;
  // fp32 accumulator, B MN-major (transpose bit 16), N = BN, M = 256
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (1u << 16) | (static_cast<uint32_t>(a.BN >> 3) << 17) |
            ((256u >> 4) << 24);
  a.tmem_cols = next_pow2_cols(static_cast<uint32_t>(2 * a.BN));
  a.timeout_ns = kWaitTimeoutNs;
  ctas = 2 * std::min(a.total_tiles, sms / 2);
  smem = static_cast<size_t>(a.stages) * a.stage_bytes + 1024 + sizeof(TcSmemTail) + 64;
  return CONV_OK;
}

int launch_tconv(const Problem& P, const void* x, const void* w, void* y, cudaStream_t st, int dev, int sms) {
  TconvArgs a;
  int ctas = 0;
  size_t smem = 0;
  int rc = plan_tconv(P, sms, a, ctas, smem);
  if (rc != CONV_OK) return rc;
  rc = set_kernel_attrs(dev);
  if (rc != CONV_OK) return rc;
  a.y = y;
  const unsigned long long stall_ns = g_inject_stall_ns.exchange(0);
  if (stall_ns != 0) {
    a.inject_stall = 1;
    a.timeout_ns = stall_ns;
  }
  const DriverFns& drv = driver_fns();
  if (!drv.tiled || !drv.im2col) return CONV_EDRIVER;
  const CUtensorMapDataType dt = P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t eb = 2;
  CUtensorMap mx, mw;
  std::memset(&mx, 0, sizeof(mx));
  std::memset(&mw, 0, sizeof(mw));
  // x: the shared im2col walk of Tm pixels per dimension from the lower corner, stride 1
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  int lower[3], upper[3];
  const int rank = a.rank5 ? 5 : 4;
  gdim[0] = P.C; gdim[1] = P.W; gdim[2] = P.H;
  gstr[0] = eb * P.C;
  gstr[1] = gstr[0] * P.W;
  gstr[2] = gstr[1] * P.H;
  lower[0] = a.lower[2]; upper[0] = a.Tm[2] - P.W + a.lower[2];
  lower[1] = a.lower[1]; upper[1] = a.Tm[1] - P.H + a.lower[1];
  if (rank == 5) {
    gdim[3] = P.D; gdim[4] = P.N;
    gstr[3] = gstr[2] * P.D;
    lower[2] = a.lower[0]; upper[2] = a.Tm[0] - P.D + a.lower[0];
  } else {
    gdim[3] = P.N;
  }
  CUresult r = drv.im2col(&mx, dt, rank, const_cast<void*>(x), gdim, gstr, lower, upper, 64u,
                          static_cast<cuuint32_t>(kBM), estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(mx, P.x_bytes, drv.driver_version);
  // w [Cin][taps][Cout/G] as (co, tap, ci): boxes of 64 co x 1 tap x 64 ci
  const cuuint64_t taps = static_cast<cuuint64_t>(P.kD) * P.kH * P.kW;
  cuuint64_t wdim[3] = {static_cast<cuuint64_t>(P.Og), taps, static_cast<cuuint64_t>(P.C)};
  cuuint64_t wstr[2] = {eb * P.Og, eb * P.Og * taps};
  cuuint32_t wbox[3] = {64u, 1u, static_cast<cuuint32_t>(a.kc)};
  cuuint32_t west[3] = {1, 1, 1};
  r = drv.tiled(&mw, dt, 3, const_cast<void*>(w), wdim, wstr, wbox, west, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(mw, P.w_bytes, drv.driver_version);

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(kTcvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, conv_tconv_pair_kernel<false>, &cfg) != cudaSuccess || clusters <= 0)
    return CONV_ELAUNCH;
  cfg.gridDim = dim3(2 * std::min(ctas / 2, clusters));
  add_pdl(cfg, attr);
  const cudaError_t e = P.dtype == CONV_BF16 ? cudaLaunchKernelEx(&cfg, conv_tconv_pair_kernel<true>, mx, mw, a)
                                             : cudaLaunchKernelEx(&cfg, conv_tconv_pair_kernel<false>, mx, mw, a);
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

// Staged kernel (conv_staged.cuh) for channel counts that TMA cannot address:
// f16/bf16, one group, stride 1, O <= 128, no flip, a forward (undilated)
// input.  The block height is the multiple of 4 up to 32 that wastes the
// fewest rows of Ho (ties to the taller block); the pipeline takes as many
// slots (weights of the kH*kW taps + two region planes) as shared memory holds.
// Raw mode: 16-byte shared-memory wavefronts of one pass of the builders'
// region loads when region unit q reads pixel (q * stride) mod (Hr*Wr), from
// rows rx_row bytes apart with pixels 2C bytes apart: per 8-lane phase of a
// warp, the most distinct 128-byte lines that fall in one 16-byte bank group.
long long staged_region_wavefronts(int C, int Hr, int Wr, long long rx_row, int stride) {
  const int npix = Hr * Wr, nB = 2 * npix;
  long long total = 0;
  for (int base = 0; base < nB; base += 8) {
    for (int half = 0; half < 2; ++half) {
      long long line[8][8];
      int nl[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int l = 0; l < 8 && base + l < nB; ++l) {
        const int u = base + l, kk = u & 1;
        const int pix = static_cast<int>((static_cast<long long>(u >> 1) * stride) % npix);
        const int r = pix / Wr, c = pix - r * Wr;
        const long long src = r * rx_row + 2LL * (static_cast<long long>(c) * C + kk * 8);
        const long long blk = (src >> 4) + half;
        const int g = static_cast<int>(blk & 7);
        bool seen = false;
        for (int k = 0; k < nl[g]; ++k) seen = seen || line[g][k] == (blk >> 3);
        if (!seen) line[g][nl[g]++] = blk >> 3;
      }
      int worst = 0;
      for (int g = 0; g < 8; ++g) worst = std::max(worst, nl[g]);
      total += worst;
    }
  }
  return total;
}

int plan_staged(const Problem& P, int sms, StArgs& a, int& ctas, size_t& smem) {
  if (P.dtype == CONV_F32 || P.G != 1 || P.flip || !plain_input(P)) return CONV_EUNSUPPORTED;
  if (P.s[0] != 1 || P.s[1] != 1 || P.s[2] != 1 || P.O > 128) return CONV_EUNSUPPORTED;
  int bh = 32;
  long long best = -1;
  for (int h = 32; h >= 4; h -= 4) {
    const long long covered = static_cast<long long>((P.Ho + h - 1) / h) * h;
    if (best < 0 || covered < best) {
      best = covered;
      bh = h;
    }
  }
  const long long Hr = bh + static_cast<long long>(P.d[1]) * (P.kH - 1);
  const long long Wr = kStBlockW + static_cast<long long>(P.d[2]) * (P.kW - 1);
  const long long plane = Hr * Wr * 16;
  const long long groups = (P.O + 7) / 8;
  const long long abytes = static_cast<long long>(P.kH) * P.kW * groups * kStAGroupBytes + (16 - groups) * kStAGroupBytes;
  const long long stage = (abytes + 2 * plane + 127) / 128 * 128;
  const long long budget = static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(StTail)) - 64;
  long long nst = std::min<long long>(kMaxStages, budget / stage);
  if (nst < 2) return CONV_EUNSUPPORTED;
  // raw mode when the staged input rows and weight rows fit beside two slots:
  // a row's 16-byte cover is at most its bytes + 30
  const long long taps_hw = static_cast<long long>(P.kH) * P.kW;
  // rows 16 bytes past a multiple of 128 apart, so that eight consecutive
  // rows' 16-byte reads fall in different banks
  const long long rx_row = (Wr * P.C * 2 + 30 + 127) / 128 * 128 + 16;
  const long long rw_row = (taps_hw * P.C * 2 + 30 + 127) / 128 * 128 + 16;
  const long long raw_bytes = Hr * rx_row + static_cast<long long>(P.O) * rw_row;
  // (and each builder thread has at most kStBatch units a slot, decoded once per (block, kd))
  const long long units = 2 * Hr * Wr + taps_hw * P.O * 2;
  const bool raw = budget - raw_bytes >= 2 * stage && units <= static_cast<long long>(kStBatch) * kStBuilders;
  if (raw) nst = std::min<long long>(kMaxStages, (budget - raw_bytes) / stage);
  const long long tiles_h = (P.Ho + bh - 1) / bh, tiles_w = (P.Wo + kStBlockW - 1) / kStBlockW;
  const long long total = static_cast<long long>(P.N) * P.Do * tiles_h * tiles_w;
  if (total > 0x7fffffffLL) return CONV_EINVAL;
  std::memset(&a, 0, sizeof(a));
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C; a.O = P.O;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.K = P.K;
  a.x_blocks = static_cast<long long>((P.x_bytes + 15) / 16);
  a.w_blocks = static_cast<long long>((P.w_bytes + 15) / 16);
  a.tile_h = bh;
  a.tiles_h = static_cast<int>(tiles_h);
  a.tiles_w = static_cast<int>(tiles_w);
  a.total_tiles = static_cast<int>(total);
  a.nc16 = (P.C + 15) / 16;
  // raw mode: the pixel stride whose region loads take the fewest wavefronts
  // (ties to 1): 13 for 65 channels (10-pixel rows), 1 for 21 or 3
  a.pix_stride = 1;
  if (raw) {
    long long best_w = staged_region_wavefronts(P.C, static_cast<int>(Hr), static_cast<int>(Wr), rx_row, 1);
    for (int st : {3, 5, 7, 9, 11, 13, 15, 17}) {
      if (std::gcd(static_cast<long long>(st), Hr * Wr) != 1) continue;
      const long long wv = staged_region_wavefronts(P.C, static_cast<int>(Hr), static_cast<int>(Wr), rx_row, st);
      if (wv < best_w) {
        best_w = wv;
        a.pix_stride = st;
      }
    }
  }
  a.Hr = static_cast<int>(Hr);
  a.Wr = static_cast<int>(Wr);
  a.plane_bytes = static_cast<uint32_t>(plane);
  a.tap_bytes = static_cast<uint32_t>(groups * kStAGroupBytes);
  a.a_bytes = static_cast<uint32_t>(abytes);
  a.stage_bytes = static_cast<uint32_t>(stage);
  a.stages = static_cast<int>(nst);
  a.raw = raw ? 1 : 0;
  a.rx_row = static_cast<uint32_t>(rx_row);
  a.rw_row = static_cast<uint32_t>(rw_row);
  a.raw_x_off = static_cast<uint32_t>(nst * stage);
  a.raw_w_off = a.raw_x_off + static_cast<uint32_t>(Hr * rx_row);
  a.tail_off = static_cast<uint32_t>(nst * stage + (raw ? raw_bytes : 0));
  const uint32_t ab = P.dtype == CONV_BF16 ? 1u : 0u;
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (static_cast<uint32_t>(kStBlockW * bh >> 3) << 17) |
            ((128u >> 4) << 24);
  a.tmem_cols = 2 * kStAccStride;
  a.timeout_ns = kWaitTimeoutNs;
  ctas = static_cast<int>(std::min<long long>(total, sms));
  smem = static_cast<size_t>(a.tail_off) + 1024 + sizeof(StTail) + 64;
  return CONV_OK;
}

int launch_staged(const Problem& P, const void* x, const void* w, void* y, cudaStream_t st, int dev, int sms) {
  StArgs a;
  int ctas = 0;
  size_t smem = 0;
  int rc = plan_staged(P, sms, a, ctas, smem);
  if (rc != CONV_OK) return rc;
  rc = set_kernel_attrs(dev);
  if (rc != CONV_OK) return rc;
  a.x = x;
  a.w = w;
  a.y = y;
  const unsigned long long stall_ns = g_inject_stall_ns.exchange(0);
  if (stall_ns != 0) {
    a.inject_stall = 1;
    a.timeout_ns = stall_ns;
  }
  const bool bf = P.dtype == CONV_BF16, k33 = P.kH == 3 && P.kW == 3;
  auto* k = conv_fwd_tc_staged_kernel<false, 0, 0, false>;  // every instantiation has this signature
  if (a.raw)
    k = bf ? (k33 ? conv_fwd_tc_staged_kernel<true, 3, 3, true> : conv_fwd_tc_staged_kernel<true, 0, 0, true>)
           : (k33 ? conv_fwd_tc_staged_kernel<false, 3, 3, true> : conv_fwd_tc_staged_kernel<false, 0, 0, true>);
  else
    k = bf ? (k33 ? conv_fwd_tc_staged_kernel<true, 3, 3, false> : conv_fwd_tc_staged_kernel<true, 0, 0, false>)
           : (k33 ? conv_fwd_tc_staged_kernel<false, 3, 3, false> : conv_fwd_tc_staged_kernel<false, 0, 0, false>);
  const cudaError_t e = launch_pdl(k, dim3(ctas), dim3(kStThreads), smem, st, 1, a);
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

int choose_variant(const Problem& P, int sms) {
  if (!plain_input(P)) {
    if (P.dtype == CONV_F32) return CONV_VARIANT_SIMT;
    TconvArgs ta;
    int c;
    size_t sm;
    return plan_tconv(P, sms, ta, c, sm) == CONV_OK ? CONV_VARIANT_TC_TMA_PHASES : CONV_VARIANT_TC_GATHER;
  }
  if (dw_fits(P)) return CONV_VARIANT_DEPTHWISE;
  if (P.dtype == CONV_F32) return CONV_VARIANT_SIMT;
  bool r5;
  if (!tma_fits(P, r5)) {
    TcPlan pp;
    if (plan_phase(P, sms, pp) == CONV_OK) return CONV_VARIANT_TC_PHASE;
    // the staged kernel from 16 channels a group up ((4,32^3,65)->65: 0.153
    // against 0.531 ms; 21 channels: 0.0193 against 0.0201); below that its
    // fixed per-slot cost loses to the gather kernel (3 channels: 0.0170
    // against 0.0087 ms)
    StArgs sa;
    int c;
    size_t sm;
    return P.Cg >= 16 && plan_staged(P, sms, sa, c, sm) == CONV_OK ? CONV_VARIANT_TC_STAGED : CONV_VARIANT_TC_GATHER;
  }
  if (P.Og % 64 == 0 && P.Og % 256 != 0 && P.kH >= 2) {
    TcPlan hp;
    if (plan_halo_t(P, false, sms, hp) == CONV_OK && hp.args.total_tiles >= sms) return CONV_VARIANT_TC_HALO_T;
  }
  // short reductions (K <= 256, e.g. 3x1x1 over 64 channels): the plain
  // single-CTA kernel with its TMA-store epilogue (3x1x1 64->128: 0.0178 ms
  // against 0.0197 for the transposed kernel)
  if (P.Og % kTO == 0 && P.Og % 256 != 0 && P.K <= 256 && P.O % 8 == 0) return CONV_VARIANT_TC_TMA;
  if (P.Og % kTO == 0 && P.Og % 256 != 0 && P.M <= 0x7fffffffLL - 256 &&
      (P.M + 255) / 256 * (P.Og / kTO) * P.G >= sms)
    return CONV_VARIANT_TC_TMA_T;
  const long long og_tiles = (P.Og + 255) / 256;
  const long long pair_tiles = (P.M + 2 * kBM - 1) / (2 * kBM) * og_tiles * P.G;
  return pair_tiles >= sms / 2 ? CONV_VARIANT_TC_TMA_PAIR : CONV_VARIANT_TC_TMA;
}

// ---------------------------------------------------------------- launches

// y viewed as [M, O] (O innermost) for the transposed kernel's TMA stores:
// boxes of 128 channels x 32 pixels, rows beyond M clipped.
int encode_y_map(const Problem& P, void* y, CUtensorMap& my) {
  std::memset(&my, 0, sizeof(my));
  const DriverFns& drv = driver_fns();
  if (!drv.tiled) return CONV_EDRIVER;
  const CUtensorMapDataType dt =
      P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  cuuint64_t dim[2] = {static_cast<cuuint64_t>(P.O), static_cast<cuuint64_t>(P.M)};
  cuuint64_t str[1] = {static_cast<cuuint64_t>(P.O) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kTO), static_cast<cuuint32_t>(kTEpiRows)};
  cuuint32_t est[2] = {1, 1};
  const CUresult r = drv.tiled(&my, dt, 2, y, dim, str, box, est, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(my, static_cast<size_t>(P.M) * P.O * 2, drv.driver_version);
  return CONV_OK;
}

// y viewed as [M, O] for the plain-orientation kernels' TMA stores: boxes of
// 32 channels x 32 pixel rows in the 64-byte swizzle pattern, rows beyond M
// and channels beyond O clipped.
int encode_y_rows_map(const Problem& P, void* y, CUtensorMap& my) {
  std::memset(&my, 0, sizeof(my));
  const DriverFns& drv = driver_fns();
  if (!drv.tiled) return CONV_EDRIVER;
  const CUtensorMapDataType dt =
      P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  cuuint64_t dim[2] = {static_cast<cuuint64_t>(P.O), static_cast<cuuint64_t>(P.M)};
  cuuint64_t str[1] = {static_cast<cuuint64_t>(P.O) * 2};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t est[2] = {1, 1};
  const CUresult r = drv.tiled(&my, dt, 2, y, dim, str, box, est, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(my, static_cast<size_t>(P.M) * P.O * 2, drv.driver_version);
  return CONV_OK;
}

// y viewed as [N, (Do,) Ho, Wo, O] for the transposed halo kernel's TMA
// stores: boxes of mo/4 channels (one epilogue warp's quarter of the tile's
// 64 or 128) x 8 columns x 4 rows, clipped at the edges.
int encode_y_block_map(const Problem& P, bool rank5, int mo, void* y, CUtensorMap& my) {
  std::memset(&my, 0, sizeof(my));
  const DriverFns& drv = driver_fns();
  if (!drv.tiled) return CONV_EDRIVER;
  const CUtensorMapDataType dt =
      P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t eb = 2;
  cuuint64_t dim[5] = {static_cast<cuuint64_t>(P.O), static_cast<cuuint64_t>(P.Wo), static_cast<cuuint64_t>(P.Ho),
                       static_cast<cuuint64_t>(rank5 ? P.Do : P.N), static_cast<cuuint64_t>(P.N)};
  cuuint64_t str[4] = {eb * P.O, eb * P.O * P.Wo, eb * P.O * P.Wo * P.Ho, eb * P.O * P.Wo * P.Ho * P.Do};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(mo / 4), static_cast<cuuint32_t>(kHTBlockW),
                       static_cast<cuuint32_t>(kTEpiRows / kHTBlockW), 1u, 1u};
  cuuint32_t est[5] = {1, 1, 1, 1, 1};
  const CUresult r = drv.tiled(&my, dt, rank5 ? 5 : 4, y, dim, str, box, est, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(my, static_cast<size_t>(P.M) * P.O * 2, drv.driver_version);
  return CONV_OK;
}

int encode_maps(const Problem& P, const TcArgs& a, bool pair, bool halo, const void* x, const void* w,
                CUtensorMap& mx, CUtensorMap& mw, int w_rows = 0) {
  std::memset(&mx, 0, sizeof(mx));
  std::memset(&mw, 0, sizeof(mw));
  if (a.cchunks == 0 && a.gather_mode == GATHER_ROWS) {
    // x viewed as [N*H][W*C / box_e][box_e]; one box of stage_rows whole rows, zero fill
    const DriverFns& drv = driver_fns();
    if (!drv.tiled) return CONV_EDRIVER;
    const CUtensorMapDataType dt =
        P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t rdim[3] = {static_cast<cuuint64_t>(a.box_e), static_cast<cuuint64_t>(a.n_boxes),
                          static_cast<cuuint64_t>(P.N) * P.H};
    cuuint64_t rstr[2] = {static_cast<cuuint64_t>(a.box_e) * 2, static_cast<cuuint64_t>(P.W) * P.C * 2};
    cuuint32_t rbox[3] = {static_cast<cuuint32_t>(a.box_e), static_cast<cuuint32_t>(a.n_boxes),
                          static_cast<cuuint32_t>(a.stage_rows)};
    cuuint32_t rest[3] = {1, 1, 1};
    const CUresult r = drv.tiled(&mx, dt, 3, const_cast<void*>(x), rdim, rstr, rbox, rest,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return CONV_EDRIVER;
    small_tensor_fixup(mx, P.x_bytes, drv.driver_version);
    return CONV_OK;
  }
  if (a.cchunks == 0) return CONV_OK;  // other gather modes: maps unused
  const DriverFns& drv = driver_fns();
  if (!drv.tiled || !drv.im2col) return CONV_EDRIVER;
  const CUtensorMapDataType dt =
      P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUtensorMapSwizzle swz = a.kc == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                            : (a.kc == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  // x: dims innermost first (C, W, H[, D], N)
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t estr[5];
  int lower[3], upper[3];
  const int rank = a.rank5 ? 5 : 4;
  const cuuint64_t eb = 2;
  gdim[0] = P.C; gdim[1] = P.W; gdim[2] = P.H;
  gstr[0] = eb * P.C;
  gstr[1] = gstr[0] * P.W;
  gstr[2] = gstr[1] * P.H;
  estr[0] = 1; estr[1] = P.s[2]; estr[2] = P.s[1];
  lower[0] = -P.p[2]; upper[0] = P.p_hi[2] - P.d[2] * (P.kW - 1);
  lower[1] = -P.p[1]; upper[1] = P.p_hi[1] - P.d[1] * (P.kH - 1);
  if (rank == 5) {
    gdim[3] = P.D; gdim[4] = P.N;
    gstr[3] = gstr[2] * P.D;
    estr[3] = P.s[0]; estr[4] = 1;
    lower[2] = -P.p[0]; upper[2] = P.p_hi[0] - P.d[0] * (P.kD - 1);
  } else {
    gdim[3] = P.N;
    estr[3] = 1;
  }
  CUresult r;
  if (halo) {
    // a tiled box of kc channels x halo_w x halo_h pixels (x 1 depth) x 1 image
    cuuint32_t hbox[5] = {static_cast<cuuint32_t>(a.kc), static_cast<cuuint32_t>(a.halo_w),
                          static_cast<cuuint32_t>(a.halo_h), 1u, 1u};
    cuuint32_t hest[5] = {1u, 1u, 1u, 1u, 1u};
    r = drv.tiled(&mx, dt, rank, const_cast<void*>(x), gdim, gstr, hbox, hest, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    r = drv.im2col(&mx, dt, rank, const_cast<void*>(x), gdim, gstr, lower, upper, static_cast<cuuint32_t>(a.kc),
                   static_cast<cuuint32_t>(kBM), estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(mx, P.x_bytes, drv.driver_version);
  // w viewed as [O, K] (K innermost)
  cuuint64_t wdim[2] = {static_cast<cuuint64_t>(P.K), static_cast<cuuint64_t>(P.O)};
  cuuint64_t wstr[1] = {static_cast<cuuint64_t>(P.K) * eb};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(a.kc),
                       static_cast<cuuint32_t>(w_rows > 0 ? w_rows : (pair ? a.BN / 2 : a.BN))};
  cuuint32_t west[2] = {1, 1};
  r = drv.tiled(&mw, dt, 2, const_cast<void*>(w), wdim, wstr, box, west, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(mw, P.w_bytes, drv.driver_version);
  return CONV_OK;
}


// Tensor maps of the phase-packed kernel: overlapping input windows (rows
// pitch elements apart, inside the input row), plain input rows for the edge
// windows, and y as [N, Ho, Wo/P, P*O].
int encode_phase_maps(const Problem& P, const TcArgs& a, const void* x, void* y, CUtensorMap& min_,
                      CUtensorMap& medge, CUtensorMap& my) {
  std::memset(&min_, 0, sizeof(min_));
  std::memset(&medge, 0, sizeof(medge));
  std::memset(&my, 0, sizeof(my));
  const DriverFns& drv = driver_fns();
  if (!drv.tiled) return CONV_EDRIVER;
  const CUtensorMapDataType dt =
      P.dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t eb = 2, WC = static_cast<cuuint64_t>(P.W) * P.C;
  const cuuint64_t sh = static_cast<cuuint64_t>(P.s[1]);
  const cuuint64_t pitch = static_cast<cuuint64_t>(a.ph_P) * P.s[2] * P.C;
  cuuint32_t est[5] = {1, 1, 1, 1, 1};
  {
    const char* base = static_cast<const char*>(x) + eb * (pitch * a.ph_nleft - a.ph_align);
    cuuint64_t dim[5] = {static_cast<cuuint64_t>(kPhWin), static_cast<cuuint64_t>(a.ph_qint), sh,
                         static_cast<cuuint64_t>(P.H) / sh, static_cast<cuuint64_t>(P.N)};
    cuuint64_t str[4] = {eb * pitch, eb * WC, eb * WC * sh, eb * WC * P.H};
    cuuint32_t box[5] = {static_cast<cuuint32_t>(kPhWin), static_cast<cuuint32_t>(a.ph_qint), 1u,
                         static_cast<cuuint32_t>(a.ph_rows), 1u};
    const CUresult r = drv.tiled(&min_, dt, 5, const_cast<char*>(base), dim, str, box, est,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return CONV_EDRIVER;
    small_tensor_fixup(min_, P.x_bytes, drv.driver_version);
  }
  {
    cuuint64_t dim[4] = {WC, sh, static_cast<cuuint64_t>(P.H) / sh, static_cast<cuuint64_t>(P.N)};
    cuuint64_t str[3] = {eb * WC, eb * WC * sh, eb * WC * P.H};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(kPhWin), 1u, static_cast<cuuint32_t>(a.ph_rows), 1u};
    const CUresult r = drv.tiled(&medge, dt, 4, const_cast<void*>(x), dim, str, box, est,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return CONV_EDRIVER;
    small_tensor_fixup(medge, P.x_bytes, drv.driver_version);
  }
  {
    const cuuint64_t row = static_cast<cuuint64_t>(a.BN);  // P*O elements per GEMM row
    cuuint64_t dim[4] = {row, static_cast<cuuint64_t>(a.ph_qtot), static_cast<cuuint64_t>(P.Ho),
                         static_cast<cuuint64_t>(P.N)};
    cuuint64_t str[3] = {eb * row, eb * row * a.ph_qtot, eb * row * a.ph_qtot * P.Ho};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(a.ph_gcols), static_cast<cuuint32_t>(a.ph_qtot),
                         static_cast<cuuint32_t>(a.ph_rows), 1u};
    const CUresult r = drv.tiled(&my, dt, 4, y, dim, str, box, est, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 a.ph_gcols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                 CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return CONV_EDRIVER;
    small_tensor_fixup(my, P.y_bytes, drv.driver_version);
  }
  return CONV_OK;
}

int launch_tc(const Problem& P, const TcPlan& plan, const void* x, const void* w, void* y, cudaStream_t st,
              int dev) {
  int rc = set_kernel_attrs(dev);
  if (rc != CONV_OK) return rc;
  TcArgs a = plan.args;
  a.x = x; a.w = w; a.y = y;
  a.flip = P.flip;
  a.taps = P.kD * P.kH * P.kW;
  const unsigned long long stall_ns = g_inject_stall_ns.exchange(0);
  if (stall_ns != 0) {
    a.inject_stall = 1;
    a.timeout_ns = stall_ns;
  }
  CUtensorMap mx, mw;
  const bool halo = plan.variant == CONV_VARIANT_TC_HALO || plan.variant == CONV_VARIANT_TC_HALO_PAIR;
  if (plan.variant == CONV_VARIANT_TC_PHASE) {
    CUtensorMap me, my;
    rc = encode_phase_maps(P, a, x, y, mx, me, my);
    if (rc != CONV_OK) return rc;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(plan.ctas);
    cfg.blockDim = dim3(kPhThreads);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // never launch more pairs than can be resident together
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, conv_fwd_tc_phase_kernel<false>, &cfg) != cudaSuccess ||
        clusters <= 0)
      return CONV_ELAUNCH;
    cfg.gridDim = dim3(2 * std::min(plan.ctas / 2, clusters));
    add_pdl(cfg, attr);
    const cudaError_t e = P.dtype == CONV_BF16 ? cudaLaunchKernelEx(&cfg, conv_fwd_tc_phase_kernel<true>, mx, me, my, a)
                                               : cudaLaunchKernelEx(&cfg, conv_fwd_tc_phase_kernel<false>, mx, me, my, a);
    return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
  }
  if (plan.variant == CONV_VARIANT_TC_HALO_T || plan.variant == CONV_VARIANT_TC_HALO_T_PAIR) {
    CUtensorMap my;
    rc = encode_maps(P, a, false, true, x, w, mx, mw, a.mo);
    if (rc == CONV_OK) rc = encode_y_block_map(P, a.rank5 != 0, a.mo, y, my);
    if (rc != CONV_OK) return rc;
    const bool bf = P.dtype == CONV_BF16;
    if (!plan.pair) {
      const cudaError_t e1 = launch_pdl(bf ? conv_fwd_tc_halo_t_kernel<true, false> : conv_fwd_tc_halo_t_kernel<false, false>,
                                        dim3(plan.ctas), dim3(kTThreads), plan.smem, st, 1, mx, mw, my, a);
      return e1 == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(plan.ctas);
    cfg.blockDim = dim3(kTThreads);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // never launch more pairs than can be resident together
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, conv_fwd_tc_halo_t_kernel<false, true>, &cfg) != cudaSuccess ||
        clusters <= 0)
      return CONV_ELAUNCH;
    cfg.gridDim = dim3(2 * std::min(plan.ctas / 2, clusters));
    add_pdl(cfg, attr);
    const cudaError_t e = bf ? cudaLaunchKernelEx(&cfg, conv_fwd_tc_halo_t_kernel<true, true>, mx, mw, my, a)
                             : cudaLaunchKernelEx(&cfg, conv_fwd_tc_halo_t_kernel<false, true>, mx, mw, my, a);
    return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
  }
  if (plan.variant == CONV_VARIANT_TC_TMA_T) {
    CUtensorMap my;
    rc = encode_maps(P, a, false, false, x, w, mx, mw, kTO);
    if (rc == CONV_OK) rc = encode_y_map(P, y, my);
    if (rc != CONV_OK) return rc;
    const cudaError_t e = launch_pdl(P.dtype == CONV_BF16 ? conv_fwd_tc_t_kernel<true> : conv_fwd_tc_t_kernel<false>,
                                     dim3(plan.ctas), dim3(kTTileThreads), plan.smem, st, 1, mx, mw, my, a);
    return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
  }
  rc = encode_maps(P, a, plan.pair, halo, x, w, mx, mw);
  if (rc != CONV_OK) return rc;
  CUtensorMap my;
  std::memset(&my, 0, sizeof(my));
  if (a.y_tma) {
    rc = encode_y_rows_map(P, y, my);
    if (rc != CONV_OK) return rc;
  }
  const dim3 grid(plan.ctas), block(plan.variant == CONV_VARIANT_TC_TMA ? tc_threads<MODE_TMA>()
                                                                         : tc_threads<MODE_GATHER>());
  const bool bf = P.dtype == CONV_BF16;
  if (halo && !plan.pair) {
    const cudaError_t e = launch_pdl(bf ? conv_fwd_tc_halo_kernel<true, false> : conv_fwd_tc_halo_kernel<false, false>,
                                     grid, dim3(192), plan.smem, st, 1, mx, mw, a);
    return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
  }
  if (plan.pair) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(plan.ctas);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // never launch more pairs than can be resident together (a second,
    // partial wave of pairs would double the tail)
    int clusters = 0;
    {
      const int slot = (halo ? 2 : 0) + (bf ? 1 : 0);
      std::lock_guard<std::mutex> lk(g_mu);
      if (g_dev[dev].pair_smem[slot] != plan.smem) {
        int c = 0;
        cudaError_t oe;
        if (halo)
          oe = bf ? cudaOccupancyMaxActiveClusters(&c, conv_fwd_tc_halo_kernel<true, true>, &cfg)
                  : cudaOccupancyMaxActiveClusters(&c, conv_fwd_tc_halo_kernel<false, true>, &cfg);
        else
          oe = bf ? cudaOccupancyMaxActiveClusters(&c, conv_fwd_tc_pair_kernel<true>, &cfg)
                  : cudaOccupancyMaxActiveClusters(&c, conv_fwd_tc_pair_kernel<false>, &cfg);
        if (oe != cudaSuccess || c <= 0) return CONV_ELAUNCH;
        g_dev[dev].pair_smem[slot] = plan.smem;
        g_dev[dev].pair_clusters[slot] = c;
      }
      clusters = g_dev[dev].pair_clusters[slot];
    }
    cfg.gridDim = dim3(2 * std::min(plan.ctas / 2, clusters));
    add_pdl(cfg, attr);
    cudaError_t e;
    if (halo)
      e = bf ? cudaLaunchKernelEx(&cfg, conv_fwd_tc_halo_kernel<true, true>, mx, mw, a)
             : cudaLaunchKernelEx(&cfg, conv_fwd_tc_halo_kernel<false, true>, mx, mw, a);
    else
      e = bf ? cudaLaunchKernelEx(&cfg, conv_fwd_tc_pair_kernel<true>, mx, mw, my, a)
             : cudaLaunchKernelEx(&cfg, conv_fwd_tc_pair_kernel<false>, mx, mw, my, a);
    return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
  }
  // every instantiation below has the same signature
  auto* k = bf ? conv_fwd_tc_kernel<MODE_TMA, true> : conv_fwd_tc_kernel<MODE_TMA, false>;
  if (plan.variant != CONV_VARIANT_TC_TMA) {
    if (a.tp_on)
      k = bf ? conv_fwd_tc_kernel<MODE_GATHER, true, true, true> : conv_fwd_tc_kernel<MODE_GATHER, false, true, true>;
    else if (a.idil_on || a.wtrans)
      k = bf ? conv_fwd_tc_kernel<MODE_GATHER, true, true> : conv_fwd_tc_kernel<MODE_GATHER, false, true>;
    else
      k = bf ? conv_fwd_tc_kernel<MODE_GATHER, true> : conv_fwd_tc_kernel<MODE_GATHER, false>;
  }
  const cudaError_t e = launch_pdl(k, grid, block, plan.smem, st, 1, mx, mw, my, a);
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

// SIMT tile shape: TN (channels per thread, BN = 16*TN) from {2, 4, 5, 6, 8}
// wasting the fewest padded channels of O/G (ties to the wider tile); TM = 4
// (64-pixel tiles: at most 128 registers, two CTAs per SM; 128-pixel tiles
// measured slower on B200 at 170-255 registers).  f16/bf16 (a cross-check
// path) use the 4 x 4 shape only.
struct SimtShape {
  int tm, tn;
};

SimtShape simt_shape(const Problem& P, int sms) {
  SimtShape sh{4, 4};
  if (P.dtype != CONV_F32) return sh;
  static const int kTns[5] = {8, 6, 5, 4, 2};
  long long best = -1;
  for (int tn : kTns) {
    const long long padded = static_cast<long long>((P.Og + 16 * tn - 1) / (16 * tn)) * 16 * tn;
    if (best < 0 || padded < best) {
      best = padded;
      sh.tn = tn;
    }
  }
  (void)sms;
  return sh;
}

template <typename T, int TM, bool TR, bool MASK = false>
cudaError_t launch_simt_tn(int tn, dim3 grid, cudaStream_t st, const SimtArgs& a) {
  auto* k = conv_fwd_simt_kernel<T, TM, 4, TR, MASK>;
  switch (tn) {
    case 2: k = conv_fwd_simt_kernel<T, TM, 2, TR, MASK>; break;
    case 5: k = conv_fwd_simt_kernel<T, TM, 5, TR, MASK>; break;
    case 6: k = conv_fwd_simt_kernel<T, TM, 6, TR, MASK>; break;
    case 8: k = conv_fwd_simt_kernel<T, TM, 8, TR, MASK>; break;
    default: break;
  }
  return launch_pdl(k, grid, dim3(kSimtThreads), 0, st, 1, a);
}

int launch_simt(const Problem& P, const void* x, const void* w, void* y, cudaStream_t st, int sms) {
  SimtArgs a;
  a.N = P.N; a.D = P.D; a.H = P.H; a.W = P.W; a.C = P.C; a.O = P.O;
  a.kD = P.kD; a.kH = P.kH; a.kW = P.kW;
  a.sd = P.s[0]; a.sh = P.s[1]; a.sw = P.s[2];
  a.pd = P.p[0]; a.ph = P.p[1]; a.pw = P.p[2];
  a.dd = P.d[0]; a.dh = P.d[1]; a.dw = P.d[2];
  a.G = P.G; a.Cg = P.Cg; a.Og = P.Og;
  a.Do = P.Do; a.Ho = P.Ho; a.Wo = P.Wo;
  a.M = P.M; a.K = static_cast<int>(P.K);
  a.flip = P.flip;
  a.taps = P.kD * P.kH * P.kW;
  a.idd = P.idil[0]; a.idh = P.idil[1]; a.idw = P.idil[2];
  a.wtrans = P.wtrans;
  a.x = x; a.w = w; a.y = y;
  const SimtShape sh = simt_shape(P, sms);
  const long long mt = (P.M + 16 * sh.tm - 1) / (16 * sh.tm);
  const long long nt = (P.Og + 16 * sh.tn - 1) / (16 * sh.tn);
  if (mt > 0x7fffffffLL || nt > 65535 || P.G > 65535) return CONV_EUNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(mt), static_cast<unsigned>(nt), P.G);
  cudaError_t e;
  const bool tr = !plain_input(P);
  if (P.dtype == CONV_F32) {
    // forward problems with at most 32 filter taps and at least 16 channels a
    // tap: the masked loader (its per-block mask set-up costs more than it
    // saves when K is a few steps long)
    const bool mask = !tr && a.taps <= 32 && a.Cg >= 16;
    e = tr ? launch_simt_tn<float, 4, true>(sh.tn, grid, st, a)
           : (mask ? launch_simt_tn<float, 4, false, true>(sh.tn, grid, st, a)
                   : launch_simt_tn<float, 4, false>(sh.tn, grid, st, a));
  } else if (P.dtype == CONV_F16) {
    e = launch_pdl(tr ? conv_fwd_simt_kernel<__half, 4, 4, true> : conv_fwd_simt_kernel<__half, 4, 4>, grid,
                   dim3(kSimtThreads), 0, st, 1, a);
  } else {
    e = launch_pdl(tr ? conv_fwd_simt_kernel<__nv_bfloat16, 4, 4, true> : conv_fwd_simt_kernel<__nv_bfloat16, 4, 4>,
                   grid, dim3(kSimtThreads), 0, st, 1, a);
  }
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

// ---------------------------------------------------------------- host-buffer pipeline

// conv_fwd_host splits the batch into chunks so that the upload of chunk i+1,
// the kernel on chunk i and the download of chunk i-1 overlap (PCIe carries
// both directions at once).  Two copy streams and the events that order them
// are created once per device and kept; a mutex makes calls on one device
// take turns (the call waits for its result anyway).
constexpr int kHostMaxChunks = 16;
constexpr size_t kHostMinChunkBytes = size_t(4) << 20;

struct HostPipe {
  std::mutex mu;
  bool init = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, finished = nullptr;
  cudaEvent_t loaded[kHostMaxChunks] = {}, computed[kHostMaxChunks] = {};
};
HostPipe g_host_pipe[kMaxDevices];

int host_pipe_init(HostPipe& hp) {
  if (hp.init) return CONV_OK;
  const unsigned f = cudaEventDisableTiming;
  if (cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&hp.start, f) != cudaSuccess || cudaEventCreateWithFlags(&hp.finished, f) != cudaSuccess)
    return CONV_ELAUNCH;
  for (int i = 0; i < kHostMaxChunks; ++i)
    if (cudaEventCreateWithFlags(&hp.loaded[i], f) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.computed[i], f) != cudaSuccess)
      return CONV_ELAUNCH;
  hp.init = true;
  return CONV_OK;
}

// Chunks of whole images, at most kHostMaxChunks, each moving at least
// kHostMinChunkBytes of x and y (small problems run as one chunk), and one
// chunk when an image's bytes are not a multiple of 16.
int host_chunks(const Problem& P) {
  // chunk offsets must keep the 16-byte alignment the tensor maps need
  if ((P.x_bytes / P.N) % 16 != 0 || (P.y_bytes / P.N) % 16 != 0) return 1;
  const long long by_bytes = static_cast<long long>((P.x_bytes + P.y_bytes) / kHostMinChunkBytes);
  const long long n = std::min<long long>({static_cast<long long>(P.N), static_cast<long long>(kHostMaxChunks),
                                           std::max<long long>(1, by_bytes)});
  return static_cast<int>(std::max<long long>(1, n));
}

// Reads the device status word after the caller's stream has finished; clears
// it and returns CONV_ETIMEOUT if a kernel gave up on a pipeline wait.
int read_and_clear_status() {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_conv_status, sizeof(v)) != cudaSuccess) return CONV_ELAUNCH;
  if (v == 0) return CONV_OK;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_conv_status, &zero, sizeof(zero)) != cudaSuccess) return CONV_ELAUNCH;
  return CONV_ETIMEOUT;
}

int run(const Problem& P, const void* x, const void* w, void* y, int variant, cudaStream_t st) {
  int dev;
  int rc = current_device(dev);
  if (rc != CONV_OK) return rc;
  int sms;
  rc = device_sms(dev, sms);
  if (rc != CONV_OK) return rc;
  if (variant == CONV_VARIANT_AUTO) variant = choose_variant(P, sms);
  if (variant == CONV_VARIANT_SIMT) return launch_simt(P, x, w, y, st, sms);
  if (variant == CONV_VARIANT_DEPTHWISE) return launch_dw(P, x, w, y, st, sms);
  if (variant == CONV_VARIANT_DEPTHWISE_DIRECT) return launch_dw_direct(P, x, w, y, st);
  if (variant == CONV_VARIANT_TC_TMA_PHASES) return launch_tconv(P, x, w, y, st, dev, sms);
  if (variant == CONV_VARIANT_TC_STAGED) return launch_staged(P, x, w, y, st, dev, sms);
  TcPlan plan;
  rc = plan_tc(P, variant, sms, plan);
  if (rc != CONV_OK) return rc;
  return launch_tc(P, plan, x, w, y, st, dev);
}

// Queues conv_fwd_host's copies and kernels: the upload of chunk i on the
// upload stream, its kernel on the caller's stream, its download on the
// download stream, ordered by events; the caller's stream finally waits for
// the last download.  Returns at the first failure (work already queued stays
// queued; the caller drains the streams).
int host_pipeline(const Problem& P, HostPipe& hp, int variant, int nch, const void* x_host, const void* w_host,
                  void* y_host, void* x_dev, const void* w_dev, void* y_dev, cudaStream_t st) {
  const size_t x_img = P.x_bytes / P.N, y_img = P.y_bytes / P.N;
  const char* xh = static_cast<const char*>(x_host);
  char* yh = static_cast<char*>(y_host);
  char* xd = static_cast<char*>(x_dev);
  char* yd = static_cast<char*>(y_dev);
  const int stride[3] = {P.s[0], P.s[1], P.s[2]}, pad[3] = {P.p[0], P.p[1], P.p[2]}, dil[3] = {P.d[0], P.d[1], P.d[2]};
  // the copy streams start after the work already queued on the caller's stream
  if (cudaEventRecord(hp.start, st) != cudaSuccess || cudaStreamWaitEvent(hp.h2d, hp.start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp.d2h, hp.start, 0) != cudaSuccess)
    return CONV_ELAUNCH;
  if (cudaMemcpyAsync(const_cast<void*>(w_dev), w_host, P.w_bytes, cudaMemcpyHostToDevice, hp.h2d) != cudaSuccess)
    return CONV_ELAUNCH;
  int n0 = 0;
  for (int i = 0; i < nch; ++i) {
    const int nc = (P.N - n0) / (nch - i);
    Problem Pc;
    int rc = make_problem(Pc, nc, P.D, P.H, P.W, P.C, P.O, P.kD, P.kH, P.kW, stride, pad, pad, dil, P.G, 0, P.dtype);
    if (rc != CONV_OK) return rc;
    // input chunk i on the upload stream (after w), then the kernel on the
    // caller's stream, then the result chunk on the download stream
    if (cudaMemcpyAsync(xd + n0 * x_img, xh + n0 * x_img, nc * x_img, cudaMemcpyHostToDevice, hp.h2d) != cudaSuccess ||
        cudaEventRecord(hp.loaded[i], hp.h2d) != cudaSuccess || cudaStreamWaitEvent(st, hp.loaded[i], 0) != cudaSuccess)
      return CONV_ELAUNCH;
    rc = run(Pc, xd + n0 * x_img, w_dev, yd + n0 * y_img, variant, st);
    if (rc == CONV_EUNSUPPORTED) rc = run(Pc, xd + n0 * x_img, w_dev, yd + n0 * y_img, CONV_VARIANT_AUTO, st);
    if (rc != CONV_OK) return rc;
    if (cudaEventRecord(hp.computed[i], st) != cudaSuccess || cudaStreamWaitEvent(hp.d2h, hp.computed[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(yh + n0 * y_img, yd + n0 * y_img, nc * y_img, cudaMemcpyDeviceToHost, hp.d2h) != cudaSuccess)
      return CONV_ELAUNCH;
    n0 += nc;
  }
  if (cudaEventRecord(hp.finished, hp.d2h) != cudaSuccess || cudaStreamWaitEvent(st, hp.finished, 0) != cudaSuccess)
    return CONV_ELAUNCH;
  return CONV_OK;
}

}  // namespace
}  // namespace convfwd

// ---------------------------------------------------------------- weight gradient on the tensor cores
// (called from conv_wgrad.cu; the kernel lives in this translation unit with
// the device status word and the tensor-map helpers)

namespace convfwd {

constexpr int kWgtKbs = 1;        // 128-pixel sub-blocks per pipeline stage (8 pair MMAs, 1024 tensor cycles)
constexpr int kWgtPairs = 74;     // CTA pairs of a 148-SM B200: the split target (fixed, so the
                                  // summation order never depends on the device)

// Can the tensor-core weight gradient run this problem?  16-bit types, whole
// 256-channel output tiles and 64-channel column blocks per group, and an
// input geometry the TMA im2col unit describes (as for the forward kernels).
bool wgrad_tc_fits(const WgArgs& a, int dtype) {
  if (dtype != CONV_F16 && dtype != CONV_BF16) return false;
  if (a.Cg % 64 != 0 || a.Og % 256 != 0 || a.C % 8 != 0) return false;
  const bool rank5 = !(a.D == 1 && a.kD == 1 && a.pd == 0 && a.pd_hi == 0);
  const int lo = rank5 ? -16 : -128, hi = rank5 ? 15 : 127;
  const int s[3] = {a.sd, a.sh, a.sw}, p[3] = {a.pd, a.ph, a.pw}, ph[3] = {a.pd_hi, a.ph_hi, a.pw_hi};
  const int d[3] = {a.dd, a.dh, a.dw}, k[3] = {a.kD, a.kH, a.kW};
  for (int i = rank5 ? 0 : 1; i < 3; ++i) {
    if (s[i] > 8) return false;
    const long long lower = -p[i];
    const long long upper = static_cast<long long>(ph[i]) - static_cast<long long>(d[i]) * (k[i] - 1);
    const long long off = static_cast<long long>(d[i]) * (k[i] - 1);
    if (lower < lo || lower > hi || upper < lo || upper > hi || off > hi) return false;
  }
  return a.P + 2LL * kWgtBK * kWgtKbs * kWgtPairs < 0x7fffffffLL;
}

// Ranges of the pixel reduction for the tensor-core path (a function of the
// shape and `max_split` only): enough units for every CTA pair of a 148-SM
// B200, each range at least 8 sub-blocks (1024 pixels) long and a whole number
// of pipeline stages; no range is empty.
void wgrad_tc_split(const WgArgs& a, long long max_split, int& nsplit, int& chunk_sub) {
  const long long per_split = static_cast<long long>(a.G) * (a.Og / 256) * ((a.ncols + 255) / 256);
  const long long total_sub = (a.P + kWgtBK - 1) / kWgtBK;
  long long ns = std::max<long long>(1, kWgtPairs / per_split);
  ns = std::min<long long>(ns, std::max<long long>(1, total_sub / 8));
  ns = std::max<long long>(1, std::min<long long>(ns, max_split));
  long long cs = (total_sub + ns - 1) / ns;
  cs = (cs + kWgtKbs - 1) / kWgtKbs * kWgtKbs;
  nsplit = static_cast<int>((total_sub + cs - 1) / cs);
  chunk_sub = static_cast<int>(cs);
}

int wgrad_tc_launch(const WgArgs& w, int dtype, long long max_split, const void* x, const void* dy, float* part,
                    cudaStream_t st) {
  int dev;
  int rc = current_device(dev);
  if (rc != CONV_OK) return rc;
  rc = set_kernel_attrs(dev);
  if (rc != CONV_OK) return rc;
  WgTcArgs a;
  std::memset(&a, 0, sizeof(a));
  a.N = w.N; a.D = w.D; a.H = w.H; a.W = w.W; a.C = w.C; a.O = w.O;
  a.kD = w.kD; a.kH = w.kH; a.kW = w.kW;
  a.sd = w.sd; a.sh = w.sh; a.sw = w.sw; a.pd = w.pd; a.ph = w.ph; a.pw = w.pw;
  a.dd = w.dd; a.dh = w.dh; a.dw = w.dw;
  a.G = w.G; a.Cg = w.Cg; a.Og = w.Og; a.Do = w.Do; a.Ho = w.Ho; a.Wo = w.Wo;
  a.P = w.P;
  a.ncols = w.ncols;
  a.jtiles = (w.ncols + 255) / 256;
  a.otiles = w.Og / 256;
  wgrad_tc_split(w, max_split, a.nsplit, a.chunk_sub);
  const long long units = static_cast<long long>(a.G) * a.otiles * a.jtiles * a.nsplit;
  if (units > 0x7fffffffLL) return CONV_EUNSUPPORTED;
  a.total_units = static_cast<int>(units);
  a.kbs = kWgtKbs;
  a.stage_bytes = static_cast<uint32_t>(a.kbs) * kWgtSub;
  const long long avail = static_cast<long long>(kSmemBudget) - 1024 - static_cast<long long>(sizeof(TcSmemTail)) - 64;
  a.stages = static_cast<int>(std::min<long long>(kMaxStages, avail / a.stage_bytes));
  if (a.stages < 2) return CONV_EUNSUPPORTED;
  const uint32_t ab = dtype == CONV_BF16 ? 1u : 0u;
  // fp32 accumulator, both operands MN-major (transpose bits 15 and 16), N = 256, M = 256
  a.idesc = (1u << 4) | (ab << 7) | (ab << 10) | (1u << 15) | (1u << 16) | ((256u >> 3) << 17) | ((256u >> 4) << 24);
  a.rank5 = (w.D == 1 && w.kD == 1 && w.pd == 0 && w.pd_hi == 0) ? 0 : 1;
  a.timeout_ns = kWaitTimeoutNs;
  const unsigned long long stall_ns = g_inject_stall_ns.exchange(0);
  if (stall_ns != 0) {
    a.inject_stall = 1;
    a.timeout_ns = stall_ns;
  }
  a.part = part;

  const DriverFns& drv = driver_fns();
  if (!drv.tiled || !drv.im2col) return CONV_EDRIVER;
  const CUtensorMapDataType dt = dtype == CONV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t eb = 2;
  CUtensorMap mx, mdy;
  std::memset(&mx, 0, sizeof(mx));
  std::memset(&mdy, 0, sizeof(mdy));
  // x: im2col over the forward pass's output pixels, boxes of 64 channels x 64 pixels
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t estr[5];
  int lower[3], upper[3];
  const int rank = a.rank5 ? 5 : 4;
  gdim[0] = w.C; gdim[1] = w.W; gdim[2] = w.H;
  gstr[0] = eb * w.C;
  gstr[1] = gstr[0] * w.W;
  gstr[2] = gstr[1] * w.H;
  estr[0] = 1; estr[1] = w.sw; estr[2] = w.sh;
  lower[0] = -w.pw; upper[0] = w.pw_hi - w.dw * (w.kW - 1);
  lower[1] = -w.ph; upper[1] = w.ph_hi - w.dh * (w.kH - 1);
  if (rank == 5) {
    gdim[3] = w.D; gdim[4] = w.N;
    gstr[3] = gstr[2] * w.D;
    estr[3] = w.sd; estr[4] = 1;
    lower[2] = -w.pd; upper[2] = w.pd_hi - w.dd * (w.kD - 1);
  } else {
    gdim[3] = w.N;
    estr[3] = 1;
  }
  CUresult r = drv.im2col(&mx, dt, rank, const_cast<void*>(x), gdim, gstr, lower, upper, 64u,
                          static_cast<cuuint32_t>(kWgtBK), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  const size_t x_bytes = static_cast<size_t>(w.N) * w.D * w.H * w.W * w.C * eb;
  small_tensor_fixup(mx, x_bytes, drv.driver_version);
  // dy viewed as [P, O] (O innermost), boxes of 64 channels x 64 pixels; rows past P read zeros
  cuuint64_t ddim[2] = {static_cast<cuuint64_t>(w.O), static_cast<cuuint64_t>(w.P)};
  cuuint64_t dstr[1] = {static_cast<cuuint64_t>(w.O) * eb};
  cuuint32_t dbox[2] = {64u, static_cast<cuuint32_t>(kWgtBK)};
  cuuint32_t dest[2] = {1, 1};
  r = drv.tiled(&mdy, dt, 2, const_cast<void*>(dy), ddim, dstr, dbox, dest, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CONV_EDRIVER;
  small_tensor_fixup(mdy, static_cast<size_t>(w.P) * w.O * eb, drv.driver_version);

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  const size_t smem = static_cast<size_t>(a.stages) * a.stage_bytes + 1024 + sizeof(TcSmemTail) + 64;
  int sms = 0;
  rc = device_sms(dev, sms);
  if (rc != CONV_OK) return rc;
  cfg.gridDim = dim3(2 * std::min(a.total_units, sms / 2));
  cfg.blockDim = dim3(kWgtThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, conv_wgrad_tc_pair_kernel<false>, &cfg) != cudaSuccess ||
      clusters <= 0)
    return CONV_ELAUNCH;
  cfg.gridDim = dim3(2 * std::min(a.total_units, clusters));
  add_pdl(cfg, attr);
  const cudaError_t e = dtype == CONV_BF16 ? cudaLaunchKernelEx(&cfg, conv_wgrad_tc_pair_kernel<true>, mx, mdy, a)
                                           : cudaLaunchKernelEx(&cfg, conv_wgrad_tc_pair_kernel<false>, mx, mdy, a);
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

}  // namespace convfwd

namespace convfwd {
namespace {
int plan_problem(const Problem& P, int variant, int* bn, int* stages, int* ctas);
}  // namespace
}  // namespace convfwd

using namespace convfwd;

extern "C" {

int conv_out_dims_ex(int D, int H, int W, int kD, int kH, int kW, const int stride[3], const int pad_lo[3],
                     const int pad_hi[3], const int dil[3], int out[3]) {
  return out_dims_impl(D, H, W, kD, kH, kW, stride, pad_lo, pad_hi, dil, out);
}

int conv_out_dims(int D, int H, int W, int kD, int kH, int kW, const int stride[3], const int pad[3],
                  const int dil[3], int out[3]) {
  return out_dims_impl(D, H, W, kD, kH, kW, stride, pad, pad, dil, out);
}

int conv_fwd_ex(const void* x, const void* w, void* y, int N, int D, int H, int W, int C, int O, int kD, int kH,
                int kW, const int stride[3], const int pad_lo[3], const int pad_hi[3], const int dil[3], int groups,
                int flip, int dtype, int variant, conv_stream_t stream) {
  Problem P;
  int rc = make_problem(P, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil, groups, flip, dtype);
  if (rc != CONV_OK) return rc;
  rc = check_pointers(P, x, w, y);
  if (rc != CONV_OK) return rc;
  if (variant < CONV_VARIANT_AUTO || variant > CONV_VARIANT_TC_STAGED) return CONV_EINVAL;
  if (variant == CONV_VARIANT_TC_TMA_PHASES) return CONV_EUNSUPPORTED;  // transposed convolutions only
  return run(P, x, w, y, variant, reinterpret_cast<cudaStream_t>(stream));
}

int conv_fwd_variant(const void* x, const void* w, void* y, int N, int D, int H, int W, int C, int O, int kD,
                     int kH, int kW, const int stride[3], const int pad[3], const int dil[3], int groups,
                     int dtype, int variant, conv_stream_t stream) {
  return conv_fwd_ex(x, w, y, N, D, H, W, C, O, kD, kH, kW, stride, pad, pad, dil, groups, 0, dtype, variant,
                     stream);
}

int conv_fwd(const void* x, const void* w, void* y, int N, int D, int H, int W, int C, int O, int kD, int kH,
             int kW, const int stride[3], const int pad[3], const int dil[3], int groups, int dtype,
             conv_stream_t stream) {
  return conv_fwd_variant(x, w, y, N, D, H, W, C, O, kD, kH, kW, stride, pad, dil, groups, dtype,
                          CONV_VARIANT_AUTO, stream);
}

int conv_fwd_host(const void* x_host, const void* w_host, void* y_host, void* x_dev, void* w_dev, void* y_dev,
                  int N, int D, int H, int W, int C, int O, int kD, int kH, int kW, const int stride[3],
                  const int pad[3], const int dil[3], int groups, int dtype, conv_stream_t stream) {
  Problem P;
  int rc = make_problem(P, N, D, H, W, C, O, kD, kH, kW, stride, pad, pad, dil, groups, 0, dtype);
  if (rc != CONV_OK) return rc;
  if (!x_host || !w_host || !y_host) return CONV_EINVAL;
  rc = check_pointers(P, x_dev, w_dev, y_dev);
  if (rc != CONV_OK) return rc;
  if (overlaps(x_dev, P.x_bytes, w_dev, P.w_bytes)) return CONV_EALIAS;
  int dev;
  rc = current_device(dev);
  if (rc != CONV_OK) return rc;
  int sms;
  rc = device_sms(dev, sms);
  if (rc != CONV_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Every chunk runs the variant chosen for the whole batch, so the result is
  // the one conv_fwd gives on the same buffers.
  const int variant = choose_variant(P, sms);
  const int nch = host_chunks(P);
  HostPipe& hp = g_host_pipe[dev];
  std::lock_guard<std::mutex> lk(hp.mu);
  rc = host_pipe_init(hp);
  if (rc != CONV_OK) return rc;
  rc = host_pipeline(P, hp, variant, nch, x_host, w_host, y_host, x_dev, w_dev, y_dev, st);
  if (rc != CONV_OK) {
    // nothing queued by this call may still run once it returns: the caller
    // may free its buffers
    cudaStreamSynchronize(hp.h2d);
    cudaStreamSynchronize(hp.d2h);
    cudaStreamSynchronize(st);
    return rc;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return CONV_ELAUNCH;
  // a kernel that gave up on a pipeline wait left y partial: report it (and clear the word)
  return read_and_clear_status();
}

int conv_plan_ex(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW, const int stride[3],
                 const int pad_lo[3], const int pad_hi[3], const int dil[3], int groups, int flip, int dtype,
                 int variant, int* bn, int* stages, int* ctas) {
  Problem P;
  int rc = make_problem(P, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil, groups, flip, dtype);
  if (rc != CONV_OK) return rc;
  return plan_problem(P, variant, bn, stages, ctas);
}

int conv_transpose_out_dims(int D, int H, int W, int kD, int kH, int kW, const int stride[3], const int pad[3],
                            const int out_pad[3], const int dil[3], int out[3]) {
  return convT_dims_impl(D, H, W, kD, kH, kW, stride, pad, out_pad, dil, out);
}

int conv_transpose(const void* x, const void* w, void* y, int N, int D, int H, int W, int Cin, int Cout, int kD,
                   int kH, int kW, const int stride[3], const int pad[3], const int out_pad[3], const int dil[3],
                   int groups, int dtype, int variant, conv_stream_t stream) {
  Problem P;
  int rc = make_transpose_problem(P, N, D, H, W, Cin, Cout, kD, kH, kW, stride, pad, out_pad, dil, groups, dtype);
  if (rc != CONV_OK) return rc;
  rc = check_pointers(P, x, w, y);
  if (rc != CONV_OK) return rc;
  if (variant < CONV_VARIANT_AUTO || variant > CONV_VARIANT_TC_STAGED) return CONV_EINVAL;
  return run(P, x, w, y, variant, reinterpret_cast<cudaStream_t>(stream));
}

int conv_transpose_plan(int N, int D, int H, int W, int Cin, int Cout, int kD, int kH, int kW, const int stride[3],
                        const int pad[3], const int out_pad[3], const int dil[3], int groups, int dtype, int variant,
                        int* bn, int* stages, int* ctas) {
  Problem P;
  int rc = make_transpose_problem(P, N, D, H, W, Cin, Cout, kD, kH, kW, stride, pad, out_pad, dil, groups, dtype);
  if (rc != CONV_OK) return rc;
  return plan_problem(P, variant, bn, stages, ctas);
}

}  // extern "C"

namespace convfwd {
namespace {

int plan_problem(const Problem& P, int variant, int* bn, int* stages, int* ctas) {
  int rc;
  if (variant < CONV_VARIANT_AUTO || variant > CONV_VARIANT_TC_STAGED) return CONV_EINVAL;
  int dev, sms = 148;
  if (current_device(dev) == CONV_OK) device_sms(dev, sms);
  if (variant == CONV_VARIANT_AUTO) variant = choose_variant(P, sms);
  if (variant == CONV_VARIANT_DEPTHWISE || variant == CONV_VARIANT_DEPTHWISE_DIRECT) {
    DwTmaArgs ta;
    DwForm f;
    int tgrid;
    size_t smem;
    if (variant == CONV_VARIANT_DEPTHWISE && plan_dw_tma(P, sms, ta, f, tgrid, smem) == CONV_OK) {
      if (bn) *bn = 4;  // channels per thread
      if (stages) *stages = ta.stages;
      if (ctas) *ctas = tgrid;
      return variant;
    }
    DwArgs da;
    dim3 grid, block;
    rc = plan_dw(P, da, grid, block, smem);
    if (rc != CONV_OK) return rc;
    if (bn) *bn = dw_vec(P);
    if (stages) *stages = 1;
    if (ctas) *ctas = static_cast<int>(std::min<long long>(static_cast<long long>(grid.x) * grid.y, 0x7fffffffLL));
    return variant;
  }
  if (variant == CONV_VARIANT_TC_TMA_PHASES) {
    TconvArgs ta;
    int c;
    size_t sm;
    rc = plan_tconv(P, sms, ta, c, sm);
    if (rc != CONV_OK) return rc;
    if (bn) *bn = ta.BN;
    if (stages) *stages = ta.stages;
    if (ctas) *ctas = c;
    return variant;
  }
  if (variant == CONV_VARIANT_TC_STAGED) {
    StArgs sa;
    int c;
    size_t sm;
    rc = plan_staged(P, sms, sa, c, sm);
    if (rc != CONV_OK) return rc;
    if (bn) *bn = kStBlockW * sa.tile_h;
    if (stages) *stages = sa.stages;
    if (ctas) *ctas = c;
    return variant;
  }
  if (variant == CONV_VARIANT_SIMT) {
    const SimtShape sh = simt_shape(P, sms);
    if (bn) *bn = 16 * sh.tn;
    if (stages) *stages = 2;
    if (ctas) {
      const long long mt = (P.M + 16 * sh.tm - 1) / (16 * sh.tm);
      const long long c = mt * ((P.Og + 16 * sh.tn - 1) / (16 * sh.tn)) * P.G;
      *ctas = static_cast<int>(std::min<long long>(c, 0x7fffffffLL));
    }
    return variant;
  }
  TcPlan plan;
  rc = plan_tc(P, variant, sms, plan);
  if (rc != CONV_OK) return rc;
  if (bn) *bn = plan.args.BN;
  if (stages) *stages = plan.args.stages;
  if (ctas) *ctas = plan.ctas;
  return variant;
}

}  // namespace
}  // namespace convfwd

extern "C" {

int conv_plan_variant(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW, const int stride[3],
                      const int pad[3], const int dil[3], int groups, int dtype, int variant, int* bn,
                      int* stages, int* ctas) {
  return conv_plan_ex(N, D, H, W, C, O, kD, kH, kW, stride, pad, pad, dil, groups, 0, dtype, variant, bn, stages,
                      ctas);
}

int conv_plan(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW, const int stride[3],
              const int pad[3], const int dil[3], int groups, int dtype, int* bn, int* stages, int* ctas) {
  return conv_plan_variant(N, D, H, W, C, O, kD, kH, kW, stride, pad, dil, groups, dtype, CONV_VARIANT_AUTO, bn,
                           stages, ctas);
}

int conv_last_status(conv_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return CONV_ELAUNCH;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_conv_status, sizeof(v)) != cudaSuccess) return CONV_ELAUNCH;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_conv_status, &zero, sizeof(zero)) != cudaSuccess) return CONV_ELAUNCH;
    return CONV_ETIMEOUT;
  }
  return CONV_OK;
}

const char* conv_strerror(int code) {
  switch (code) {
    case CONV_OK: return "ok";
    case CONV_EINVAL: return "invalid argument";
    case CONV_EDTYPE: return "unknown element type";
    case CONV_EALIGN: return "buffer not 16-byte aligned";
    case CONV_EALIAS: return "output overlaps an input";
    case CONV_ELAUNCH: return "CUDA launch or copy failed";
    case CONV_ETIMEOUT: return "kernel pipeline wait timed out";
    case CONV_EUNSUPPORTED: return "variant cannot run this shape or type";
    case CONV_EDRIVER: return "TMA tensor map encoding failed";
    case CONV_ESCRATCH: return "problem needs more scratch than the library's static buffer holds";
    default: return "unknown error";
  }
}

int conv_version(void) { return kVersion; }

int conv_debug_inject_stall(unsigned long long timeout_ns) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return CONV_EINVAL;
  g_inject_stall_ns.store(timeout_ns);
  return CONV_OK;
}

}  // extern "C"
