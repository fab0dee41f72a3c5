// conv_wgrad.cu -- C ABI of the weight gradient (see conv_wgrad.cuh).
//
// A separate translation unit of libconvfwd.so: validation, the split of the
// pixel reduction across blocks, and the launches (the tensor-core kernel in
// conv_wgrad_tc.cuh or the FP32 split-K kernel, either of which
// writes one fp32 partial slice per split into a caller-provided workspace,
// then the kernel that adds the slices in split order and rounds).  The split
// count depends on the problem's shape only, so a result is the same bits on
// every run and every device.  Allocates nothing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "../../include/conv_fwd.h"
#include "conv_wgrad.cuh"
#include "launch.cuh"

// Scratch of conv_wgrad_noalloc: a fixed array in the library's own device
// image, so that entry point never allocates.  Every device that loads the
// library holds it until the process exits.
static __device__ __align__(256) float g_wgrad_static_scratch[CONV_WGRAD_STATIC_SCRATCH_BYTES / sizeof(float)];

namespace convfwd {

// The tensor-core path (conv_wgrad_tc.cuh; defined in conv_fwd.cu, which holds
// the device status word and the tensor-map helpers).
bool wgrad_tc_fits(const WgArgs& a, int dtype);
void wgrad_tc_split(const WgArgs& a, long long max_split, int& nsplit, int& chunk_sub);
int wgrad_tc_launch(const WgArgs& w, int dtype, long long max_split, const void* x, const void* dy, float* part,
                    cudaStream_t st);

namespace {

bool wg_mul_ok(long long a, long long b, long long& r) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > 0x3fffffffffffffffLL / a) return false;
  r = a * b;
  return true;
}

long long wg_extent(long long in, int k, int s, int p_lo, int p_hi, int d) {
  const long long num = in + static_cast<long long>(p_lo) + p_hi - static_cast<long long>(d) * (k - 1) - 1;
  if (num < 0) return 0;
  return num / s + 1;
}

struct WgProblem {
  WgArgs a;
  int dtype;
  size_t esize;
  size_t x_bytes, dy_bytes, dw_bytes;
  long long dw_elems;
};

int wg_make(WgProblem& q, int N, int D, int H, int W, int C, int O, int kD, int kH, int kW, const int stride[3],
            const int pad_lo[3], const int pad_hi[3], const int dil[3], int groups, int dtype) {
  if (dtype != CONV_F32 && dtype != CONV_F16 && dtype != CONV_BF16) return CONV_EDTYPE;
  if (!stride || !pad_lo || !pad_hi || !dil) return CONV_EINVAL;
  if (N <= 0 || C <= 0 || O <= 0 || groups <= 0 || C % groups != 0 || O % groups != 0) return CONV_EINVAL;
  const int in[3] = {D, H, W}, k[3] = {kD, kH, kW};
  int out[3];
  for (int i = 0; i < 3; ++i) {
    if (in[i] <= 0 || k[i] <= 0 || stride[i] <= 0 || dil[i] <= 0 || pad_lo[i] < 0 || pad_hi[i] < 0)
      return CONV_EINVAL;
    const long long e = wg_extent(in[i], k[i], stride[i], pad_lo[i], pad_hi[i], dil[i]);
    if (e <= 0 || e > 0x7fffffffLL) return CONV_EINVAL;
    out[i] = static_cast<int>(e);
  }
  WgArgs& a = q.a;
  a.N = N; a.D = D; a.H = H; a.W = W; a.C = C; a.O = O;
  a.kD = kD; a.kH = kH; a.kW = kW;
  a.sd = stride[0]; a.sh = stride[1]; a.sw = stride[2];
  a.pd = pad_lo[0]; a.ph = pad_lo[1]; a.pw = pad_lo[2];
  a.pd_hi = pad_hi[0]; a.ph_hi = pad_hi[1]; a.pw_hi = pad_hi[2];
  a.dd = dil[0]; a.dh = dil[1]; a.dw = dil[2];
  a.G = groups; a.Cg = C / groups; a.Og = O / groups;
  a.Do = out[0]; a.Ho = out[1]; a.Wo = out[2];
  long long t, nx, ny, nw;
  if (!wg_mul_ok(kD, kH, t) || !wg_mul_ok(t, kW, t) || t > 0x7fffffffLL) return CONV_EINVAL;
  a.taps = static_cast<int>(t);
  if (!wg_mul_ok(t, a.Cg, t) || t > 0x7fffffffLL) return CONV_EINVAL;
  a.ncols = static_cast<int>(t);
  if (!wg_mul_ok(N, out[0], t) || !wg_mul_ok(t, out[1], t) || !wg_mul_ok(t, out[2], a.P)) return CONV_EINVAL;
  if (!wg_mul_ok(N, D, t) || !wg_mul_ok(t, H, t) || !wg_mul_ok(t, W, t) || !wg_mul_ok(t, C, nx)) return CONV_EINVAL;
  if (!wg_mul_ok(a.P, O, ny) || !wg_mul_ok(O, a.ncols, nw)) return CONV_EINVAL;
  q.dtype = dtype;
  q.esize = dtype == CONV_F32 ? 4 : 2;
  if (nx > (1LL << 50) || ny > (1LL << 50) || nw > (1LL << 40)) return CONV_EINVAL;
  q.x_bytes = static_cast<size_t>(nx) * q.esize;
  q.dy_bytes = static_cast<size_t>(ny) * q.esize;
  q.dw_bytes = static_cast<size_t>(nw) * q.esize;
  q.dw_elems = nw;
  return CONV_OK;
}

// Splits of the pixel reduction: enough blocks for two per SM of a 148-SM
// B200 (a fixed target, so the summation order never depends on the device),
// each split at least 64 K steps (1024 pixels) long, at most `max_split`.
constexpr long long kWgTargetBlocks = 2 * 148;

void wg_split(WgArgs& a, long long max_split) {
  const long long tiles = static_cast<long long>((a.ncols + kWgBN - 1) / kWgBN) * ((a.Og + kWgBM - 1) / kWgBM) * a.G;
  const long long steps = (a.P + kWgBK - 1) / kWgBK;
  long long ns = std::max<long long>(1, (kWgTargetBlocks + tiles - 1) / tiles);
  ns = std::min<long long>(ns, std::max<long long>(1, steps / 64));
  ns = std::min<long long>(ns, 65535 / a.G);
  ns = std::min<long long>(ns, max_split);
  a.nsplit = static_cast<int>(std::max<long long>(1, ns));
  a.chunk = (steps + a.nsplit - 1) / a.nsplit * kWgBK;
}

// Ranges of the pixel reduction for the path the problem runs on: the
// tensor-core kernel for 16-bit types where it fits, else the FP32 kernel.
int wg_nsplit(const WgProblem& q, long long max_split) {
  if (wgrad_tc_fits(q.a, q.dtype)) {
    int ns = 1, cs = 1;
    wgrad_tc_split(q.a, max_split, ns, cs);
    return ns;
  }
  WgArgs a = q.a;
  wg_split(a, max_split);
  return a.nsplit;
}

size_t wg_workspace(const WgProblem& q, long long max_split = 1LL << 30) {
  return static_cast<size_t>(wg_nsplit(q, max_split)) * static_cast<size_t>(q.dw_elems) * sizeof(float);
}

bool wg_overlaps(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

// Validates the buffers and queues the partial-sum kernel (tensor cores or FP32) and the ordered sum,
// with at most `max_split` splits.
int wg_launch(const WgProblem& q, const void* x, const void* dy, void* dw, void* workspace,
              unsigned long long workspace_bytes, long long max_split, cudaStream_t st) {
  if (!x || !dy || !dw) return CONV_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy) | reinterpret_cast<uintptr_t>(dw)) & 15)
    return CONV_EALIGN;
  if (wg_overlaps(dw, q.dw_bytes, x, q.x_bytes) || wg_overlaps(dw, q.dw_bytes, dy, q.dy_bytes)) return CONV_EALIAS;
  WgArgs a = q.a;
  wg_split(a, max_split);
  const bool tc = wgrad_tc_fits(q.a, q.dtype);
  if (tc) {
    int cs = 1;
    wgrad_tc_split(q.a, max_split, a.nsplit, cs);
  }
  const size_t ws = static_cast<size_t>(a.nsplit) * static_cast<size_t>(q.dw_elems) * sizeof(float);
  if (!workspace || workspace_bytes < ws) return CONV_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) & 15) return CONV_EALIGN;
  if (wg_overlaps(workspace, ws, x, q.x_bytes) || wg_overlaps(workspace, ws, dy, q.dy_bytes) ||
      wg_overlaps(workspace, ws, dw, q.dw_bytes))
    return CONV_EALIAS;
  if ((q.dw_elems + 255) / 256 > 0x7fffffffLL) return CONV_EUNSUPPORTED;
  a.x = x;
  a.dy = dy;
  a.part = static_cast<float*>(workspace);
  const dim3 grid(static_cast<unsigned>((a.ncols + kWgBN - 1) / kWgBN), static_cast<unsigned>((a.Og + kWgBM - 1) / kWgBM),
                  static_cast<unsigned>(a.G * a.nsplit));
  if (grid.y > 65535 || grid.z > 65535) return CONV_EUNSUPPORTED;
  const int dtype = q.dtype;
  if (tc) {
    const int rc = wgrad_tc_launch(q.a, dtype, max_split, x, dy, a.part, st);
    if (rc != CONV_OK) return rc;
  } else {
    auto* k = dtype == CONV_F32 ? conv_wgrad_kernel<float>
                                : (dtype == CONV_F16 ? conv_wgrad_kernel<__half> : conv_wgrad_kernel<__nv_bfloat16>);
    if (launch_pdl(k, grid, dim3(kWgThreads), 0, st, 1, a) != cudaSuccess) return CONV_ELAUNCH;
  }
  const long long n = q.dw_elems;
  if (n % 4 == 0) {
    // four elements a thread (dw is 16-byte aligned, so every slice is when n % 4 == 0)
    const dim3 blocks4(static_cast<unsigned>((n / 4 + 255) / 256));
    cudaError_t e;
    if (dtype == CONV_F32)
      e = launch_pdl(conv_wgrad_reduce4_kernel<float>, blocks4, dim3(256), 0, st, 1, a.part, static_cast<float*>(dw),
                     n, a.nsplit);
    else if (dtype == CONV_F16)
      e = launch_pdl(conv_wgrad_reduce4_kernel<__half>, blocks4, dim3(256), 0, st, 1, a.part, static_cast<__half*>(dw),
                     n, a.nsplit);
    else
      e = launch_pdl(conv_wgrad_reduce4_kernel<__nv_bfloat16>, blocks4, dim3(256), 0, st, 1, a.part,
                     static_cast<__nv_bfloat16*>(dw), n, a.nsplit);
    return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
  }
  const dim3 blocks(static_cast<unsigned>((n + 255) / 256));
  cudaError_t e;
  if (dtype == CONV_F32)
    e = launch_pdl(conv_wgrad_reduce_kernel<float>, blocks, dim3(256), 0, st, 1, a.part, static_cast<float*>(dw), n,
                   a.nsplit);
  else if (dtype == CONV_F16)
    e = launch_pdl(conv_wgrad_reduce_kernel<__half>, blocks, dim3(256), 0, st, 1, a.part, static_cast<__half*>(dw), n,
                   a.nsplit);
  else
    e = launch_pdl(conv_wgrad_reduce_kernel<__nv_bfloat16>, blocks, dim3(256), 0, st, 1, a.part,
                   static_cast<__nv_bfloat16*>(dw), n, a.nsplit);
  return e == cudaSuccess ? CONV_OK : CONV_ELAUNCH;
}

constexpr size_t kWgStaticScratchBytes = CONV_WGRAD_STATIC_SCRATCH_BYTES;
static_assert(kWgStaticScratchBytes % 256 == 0, "static scratch size");

// The array's device address, looked up once per device.  In host code the
// array's name is only a host-side stand-in; the address a kernel may be given
// comes from cudaGetSymbolAddress with that device current.
constexpr int kWgMaxDevices = 256;
std::mutex g_static_mu;
void* g_static_addr[kWgMaxDevices] = {};

int wg_static_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kWgMaxDevices) return CONV_ELAUNCH;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_wgrad_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return CONV_ELAUNCH;
    }
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
  return CONV_OK;
}

}  // namespace
}  // namespace convfwd

using namespace convfwd;

extern "C" {

int conv_wgrad_workspace_size(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW,
                              const int stride[3], const int pad_lo[3], const int pad_hi[3], const int dil[3],
                              int groups, int dtype, unsigned long long* bytes) {
  WgProblem q;
  const int rc = wg_make(q, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil, groups, dtype);
  if (rc != CONV_OK) return rc;
  if (!bytes) return CONV_EINVAL;
  *bytes = wg_workspace(q);
  return CONV_OK;
}

int conv_wgrad_plan(int N, int D, int H, int W, int C, int O, int kD, int kH, int kW, const int stride[3],
                    const int pad_lo[3], const int pad_hi[3], const int dil[3], int groups, int dtype, int* path,
                    int* nsplit) {
  WgProblem q;
  const int rc = wg_make(q, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil, groups, dtype);
  if (rc != CONV_OK) return rc;
  if (path) *path = wgrad_tc_fits(q.a, q.dtype) ? CONV_WGRAD_TENSOR_CORES : CONV_WGRAD_FP32;
  if (nsplit) *nsplit = wg_nsplit(q, 1LL << 30);
  return CONV_OK;
}

int conv_wgrad(const void* x, const void* dy, void* dw, int N, int D, int H, int W, int C, int O, int kD, int kH,
               int kW, const int stride[3], const int pad_lo[3], const int pad_hi[3], const int dil[3], int groups,
               int dtype, void* workspace, unsigned long long workspace_bytes, conv_stream_t stream) {
  WgProblem q;
  const int rc = wg_make(q, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil, groups, dtype);
  if (rc != CONV_OK) return rc;
  return wg_launch(q, x, dy, dw, workspace, workspace_bytes, 1LL << 30, reinterpret_cast<cudaStream_t>(stream));
}

int conv_wgrad_noalloc(const void* x, const void* dy, void* dw, int N, int D, int H, int W, int C, int O, int kD,
                       int kH, int kW, const int stride[3], const int pad_lo[3], const int pad_hi[3],
                       const int dil[3], int groups, int dtype, conv_stream_t stream) {
  WgProblem q;
  const int rc = wg_make(q, N, D, H, W, C, O, kD, kH, kW, stride, pad_lo, pad_hi, dil, groups, dtype);
  if (rc != CONV_OK) return rc;
  // as many splits as the static array holds slices (fewer than conv_wgrad
  // may use, so the two can differ in the last bits)
  const size_t slice = static_cast<size_t>(q.dw_elems) * sizeof(float);
  const long long max_split = static_cast<long long>(kWgStaticScratchBytes / slice);
  if (max_split < 1) return CONV_ESCRATCH;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CONV_ELAUNCH;
  void* scratch = nullptr;
  const int r = wg_static_scratch(dev, &scratch);
  if (r != CONV_OK) return r;
  return wg_launch(q, x, dy, dw, scratch, kWgStaticScratchBytes, max_split, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
