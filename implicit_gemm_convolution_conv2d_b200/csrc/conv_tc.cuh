// conv_tc.cuh -- tcgen05 implicit-GEMM convolution forward for sm_100a.
//
// GEMM view (the "Convolutions" tutorial, section 5: convolution is a GEMM of
// the weight matrix with the patch matrix; "Implicit GEMM" computes the patch
// indices inside the kernel instead of storing the patch matrix):
//   rows    m = (n, od, oh, ow)            M = N*Do*Ho*Wo     (output pixels)
//   columns o in one group                 Og = O/G           (output channels)
//   reduce  k = (kd, kh, kw, c)            K = kD*kH*kW*Cg    (weight order)
// A[m, k] = x[n, od*sd-pd+kd*dd, oh*sh-ph+kh*dh, ow*sw-pw+kw*dw, g*Cg+c] or 0
// B[o, k] = w[g*Og+o, kd, kh, kw, c]   (the weight tensor is already [O, K])
//
// One CTA per SM walks a static list of 128 x BN output tiles.  Warp roles:
//   producer  fills a ring of shared-memory stages (A: 128 rows x 64..16
//             K-elements, B: BN rows x the same), signalling `full[s]`;
//             MODE_TMA: one thread issues a TMA im2col load (A) and a TMA tiled
//             load (B) per stage -- the hardware walks the output pixels and
//             zero-fills the halo;  MODE_GATHER: four warps compute every
//             element's address and zero-fill out-of-range taps and channels
//             themselves (any C, any stride/dilation/groups);
//   MMA       one thread issues tcgen05.mma (M=128, N=BN, K=16 per
//             instruction) into a double-buffered fp32 accumulator in tensor
//             memory and releases each stage with tcgen05.commit -> empty[s];
//   epilogue  four warps read the accumulator (tcgen05.ld, one row per thread),
//             round to f16/bf16 (nearest even) and store y, while the MMA warp
//             already accumulates the next tile into the other buffer.
//
// Every wait is bounded: after `timeout_ns` the waiting thread raises a CTA
// abort flag and the device status word; all roles then leave their loops,
// drain what they have in flight (TMA loads, MMAs), free tensor memory and
// return.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace convfwd {

constexpr int kMaxStages = 16;
constexpr int kBM = 128;

// Device status word, one per device; bit 0 = a pipeline wait timed out.
// Bits 8..15 record which wait gave up first (see WaitSite).
__device__ unsigned int g_conv_status;

enum WaitSite : unsigned {
  kSiteProducerEmpty = 1,
  kSiteMmaFull = 2,
  kSiteMmaAccEmpty = 3,
  kSiteEpiAccFull = 4,
  kSiteDrain = 5,
};

struct TcArgs {
  int N, D, H, W, C, O;
  int kD, kH, kW;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  int G, Cg, Og;
  int Do, Ho, Wo;
  long long M;
  int K;              // kD*kH*kW*Cg
  int BN;             // output-channel tile, multiple of 32, <= 256
  int stages;
  int kc;             // K elements per stage (64, 32 or 16)
  int kblocks;        // stages-worth of K per tile
  int cchunks;        // Cg / kc (TMA mode)
  int m_tiles, n_tiles, total_tiles;
  uint32_t a_bytes, b_bytes, stage_bytes;
  uint32_t layout_type;  // UMMA smem layout: 2 = 128B swizzle, 4 = 64B, 6 = 32B
  uint32_t sbo;          // bytes between 8-row groups (8 * kc * 2)
  uint32_t idesc;        // tcgen05 instruction descriptor
  uint32_t tmem_cols;
  int rank5;
  const void* x;
  const void* w;
  void* y;
  unsigned long long timeout_ns;
};

struct __align__(8) TcSmemTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

__device__ __forceinline__ void raise_timeout(volatile int* abort_flag, unsigned site) {
  *abort_flag = 1;
  atomicOr(&g_conv_status, 1u | (site << 8));
}

// Bounded wait on phase `parity` of `bar`.  Returns false if the CTA is
// aborting (another role timed out) or if this wait itself timed out.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long timeout_ns, unsigned site) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > timeout_ns) {
      raise_timeout(abort_flag, site);
      return false;
    }
  }
}

// Warp-uniform bounded wait: all 32 lanes poll and leave together, so the
// warp can go on to .sync.aligned tensor-memory loads.  A completed phase
// stays observable until this warp arrives on the matching release barrier,
// so every lane eventually sees it.
__device__ __forceinline__ bool wait_bounded_warp(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag,
                                                  unsigned long long timeout_ns, unsigned site) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    const bool done = ptx::mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    const bool aborting = *abort_flag != 0;
    const bool late = ptx::globaltimer_ns() - t0 > timeout_ns;
    const unsigned stop = __ballot_sync(0xffffffffu, aborting || late);
    if (stop) {
      if ((threadIdx.x & 31) == static_cast<unsigned>(__ffs(stop) - 1) && !aborting)
        raise_timeout(abort_flag, site);
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (used while draining).
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, unsigned long long timeout_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > timeout_ns) {
      atomicOr(&g_conv_status, 1u | (kSiteDrain << 8));
      return false;
    }
  }
  return true;
}

struct TileCoord {
  int g, mt, nt;
};

__device__ __forceinline__ TileCoord decode_tile(const TcArgs& a, int tile) {
  TileCoord t;
  const int per_group = a.m_tiles * a.n_tiles;
  t.g = tile / per_group;
  const int r = tile - t.g * per_group;
  t.mt = r / a.n_tiles;
  t.nt = r - t.mt * a.n_tiles;
  return t;
}

// Output pixel m -> (n, od, oh, ow).
__device__ __forceinline__ void decode_pixel(const TcArgs& a, long long m, int& n, int& od, int& oh,
                                             int& ow) {
  ow = static_cast<int>(m % a.Wo);
  long long q = m / a.Wo;
  oh = static_cast<int>(q % a.Ho);
  q /= a.Ho;
  od = static_cast<int>(q % a.Do);
  n = static_cast<int>(q / a.Do);
}

// Byte offset of 16-byte chunk `ch` of row `r` in a K-major tile with
// 128-byte rows and the 128B swizzle (chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw128_offset(int r, int ch) {
  return static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(ch ^ (r & 7)) << 4);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

template <bool BF16>
__device__ __forceinline__ uint16_t cvt1(float v) {
  if constexpr (BF16) {
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t*>(&h);
  } else {
    __half h = __float2half_rn(v);
    return *reinterpret_cast<uint16_t*>(&h);
  }
}

enum { MODE_TMA = 0, MODE_GATHER = 1 };

template <int MODE>
struct TcRoles;

template <>
struct TcRoles<MODE_TMA> {
  static constexpr int kProducerWarps = 1;
};
template <>
struct TcRoles<MODE_GATHER> {
  static constexpr int kProducerWarps = 4;
};

template <int MODE>
constexpr int tc_threads() {
  return (TcRoles<MODE>::kProducerWarps + 1 + 4) * 32;
}

// ----------------------------------------------------------------------------
// Gather producer: 128 threads fill one stage (A rows = threads, B rows =
// threads and threads + 128) from plain global loads with zero fill.
// Element k of a row decodes to (kd, kh, kw, c) in weight order; the decode
// is carried incrementally from element to element.
// ----------------------------------------------------------------------------
struct GatherRow {
  bool valid;
  long long xbase;  // element offset of x[n, 0, 0, 0, g*Cg]
  int id0, ih0, iw0;
  // carried decode of the next k
  int kd, kh, kw, c;
};

__device__ __forceinline__ void gather_fill_a(const TcArgs& a, GatherRow& st, int kbase,
                                              uint8_t* a_tile, int r) {
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
#pragma unroll 1
  for (int ch = 0; ch < 8; ++ch) {
    uint32_t v[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      uint32_t lohi[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = kbase + ch * 8 + e2 * 2 + h;
        uint16_t val = 0;
        if (st.valid && k < a.K) {
          const int id = st.id0 + st.kd * a.dd;
          const int ih = st.ih0 + st.kh * a.dh;
          const int iw = st.iw0 + st.kw * a.dw;
          if (static_cast<unsigned>(id) < static_cast<unsigned>(a.D) &&
              static_cast<unsigned>(ih) < static_cast<unsigned>(a.H) &&
              static_cast<unsigned>(iw) < static_cast<unsigned>(a.W)) {
            const long long off =
                st.xbase + ((static_cast<long long>(id) * a.H + ih) * a.W + iw) * a.C + st.c;
            val = __ldg(x + off);
          }
        }
        lohi[h] = val;
        // advance the carried decode to k + 1
        if (++st.c == a.Cg) {
          st.c = 0;
          if (++st.kw == a.kW) {
            st.kw = 0;
            if (++st.kh == a.kH) {
              st.kh = 0;
              ++st.kd;
            }
          }
        }
      }
      v[e2] = lohi[0] | (lohi[1] << 16);
    }
    *reinterpret_cast<uint4*>(a_tile + sw128_offset(r, ch)) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

__device__ __forceinline__ void gather_fill_b(const TcArgs& a, int g, int n0, int kbase,
                                              uint8_t* b_tile, int tid) {
  const uint16_t* __restrict__ w = static_cast<const uint16_t*>(a.w);
  const bool vec = (a.K & 7) == 0;
#pragma unroll 1
  for (int o = tid; o < a.BN; o += 128) {
    const int oc = n0 + o;
    const bool ovalid = oc < a.Og;
    const long long rowoff = static_cast<long long>(g * a.Og + oc) * a.K;
#pragma unroll 1
    for (int ch = 0; ch < 8; ++ch) {
      const int k0 = kbase + ch * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (ovalid && k0 < a.K) {
        if (vec) {
          v = __ldg(reinterpret_cast<const uint4*>(w + rowoff + k0));
        } else {
          uint32_t p[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int k = k0 + e2 * 2;
            const uint32_t lo = (k < a.K) ? __ldg(w + rowoff + k) : 0u;
            const uint32_t hi = (k + 1 < a.K) ? __ldg(w + rowoff + k + 1) : 0u;
            p[e2] = lo | (hi << 16);
          }
          v = make_uint4(p[0], p[1], p[2], p[3]);
        }
      }
      *reinterpret_cast<uint4*>(b_tile + sw128_offset(o, ch)) = v;
    }
  }
}

// ----------------------------------------------------------------------------
// The kernel.
// ----------------------------------------------------------------------------
template <int MODE, bool BF16>
__global__ void __launch_bounds__(tc_threads<MODE>(), 1)
    conv_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_w, const TcArgs a) {
  constexpr int kProdWarps = TcRoles<MODE>::kProducerWarps;
  constexpr int kMmaWarp = kProdWarps;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(smem + a.stages * a.stage_bytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->full[s]), MODE == MODE_TMA ? 1u : 128u);
      ptx::mbar_init(ptx::smem_u32(&tail->empty[s]), 1u);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&tail->acc_full[b]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->acc_empty[b]), 4u);
    }
    ptx::mbar_init(ptx::smem_u32(&tail->drain), 1u);
    tail->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (MODE == MODE_TMA && threadIdx.x == 32) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(&tail->tmem_base), a.tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;

  if (warp < kProdWarps) {
    // ------------------------------------------------------------ producer
    if constexpr (MODE == MODE_TMA) {
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        long long fills = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x) {
          const TileCoord tc = decode_tile(a, tile);
          int n, od, oh, ow;
          decode_pixel(a, static_cast<long long>(tc.mt) * kBM, n, od, oh, ow);
          const int cw = ow * a.sw - a.pw, chh = oh * a.sh - a.ph, cd = od * a.sd - a.pd;
          const int orow = tc.g * a.Og + tc.nt * a.BN;
          int tap = 0, cchunk = 0;
          for (int kb = 0; kb < a.kblocks; ++kb) {
            if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag,
                              a.timeout_ns, kSiteProducerEmpty)) {
              ok = false;
              break;
            }
            const uint32_t fb = ptx::smem_u32(&tail->full[stage]);
            ptx::mbar_arrive_expect_tx(fb, a.a_bytes + a.b_bytes);
            const uint32_t sa = ptx::smem_u32(smem + stage * a.stage_bytes);
            const uint32_t sb = sa + a.a_bytes;
            const int kw = tap % a.kW;
            const int kh = (tap / a.kW) % a.kH;
            const int kd = tap / (a.kW * a.kH);
            const int c0 = tc.g * a.Cg + cchunk * a.kc;
            if (a.rank5) {
              ptx::tma_load_im2col_5d(sa, &tmap_x, fb, c0, cw, chh, cd, n,
                                      static_cast<uint16_t>(kw * a.dw),
                                      static_cast<uint16_t>(kh * a.dh),
                                      static_cast<uint16_t>(kd * a.dd));
            } else {
              ptx::tma_load_im2col_4d(sa, &tmap_x, fb, c0, cw, chh, n,
                                      static_cast<uint16_t>(kw * a.dw),
                                      static_cast<uint16_t>(kh * a.dh));
            }
            ptx::tma_load_2d(sb, &tmap_w, fb, tap * a.Cg + cchunk * a.kc, orow);
            ++fills;
            if (++cchunk == a.cchunks) {
              cchunk = 0;
              ++tap;
            }
            if (++stage == a.stages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) {
          // drain: wait for the last armed phase of every stage ever filled
          for (int s = 0; s < a.stages; ++s) {
            const long long arms = fills / a.stages + (s < fills % a.stages ? 1 : 0);
            if (arms > 0)
              wait_drain(ptx::smem_u32(&tail->full[s]), static_cast<uint32_t>((arms - 1) & 1),
                         a.timeout_ns);
          }
        }
      }
      __syncwarp();
    } else {
      const int tid = threadIdx.x;  // 0..127
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x) {
        const TileCoord tc = decode_tile(a, tile);
        GatherRow st;
        const long long m = static_cast<long long>(tc.mt) * kBM + tid;
        st.valid = m < a.M;
        int n = 0, od = 0, oh = 0, ow = 0;
        if (st.valid) decode_pixel(a, m, n, od, oh, ow);
        st.xbase = static_cast<long long>(n) * a.D * a.H * a.W * a.C + static_cast<long long>(tc.g) * a.Cg;
        st.id0 = od * a.sd - a.pd;
        st.ih0 = oh * a.sh - a.ph;
        st.iw0 = ow * a.sw - a.pw;
        st.kd = st.kh = st.kw = st.c = 0;
        const int n0 = tc.nt * a.BN;
        for (int kb = 0; kb < a.kblocks; ++kb) {
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * a.stage_bytes;
          gather_fill_a(a, st, kb * 64, sa, tid);
          gather_fill_b(a, tc.g, n0, kb * 64, sa + a.a_bytes, tid);
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(ptx::smem_u32(&tail->full[stage]));
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int t = 0;
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x, ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag,
                          a.timeout_ns, kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        for (int kb = 0; kb < a.kblocks; ++kb) {
          if (!wait_bounded(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns,
                            kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = ptx::smem_u32(smem + stage * a.stage_bytes);
          const uint32_t sb = sa + a.a_bytes;
          const int ksteps = a.kc >> 4;
          for (int k = 0; k < ksteps; ++k) {
            const uint64_t da = ptx::smem_desc(sa + k * 32, 16, a.sbo, a.layout_type);
            const uint64_t db = ptx::smem_desc(sb + k * 32, 16, a.sbo, a.layout_type);
            ptx::mma_f16(d_tmem, da, db, a.idesc, (kb | k) != 0 ? 1u : 0u);
          }
          ptx::mma_commit(ptx::smem_u32(&tail->empty[stage]));
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) ptx::mma_commit(ptx::smem_u32(&tail->acc_full[acc]));
      }
      // every MMA this thread issued has completed once `drain` fires
      ptx::mma_commit(ptx::smem_u32(&tail->drain));
      wait_drain(ptx::smem_u32(&tail->drain), 0, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = q * 32 + lane;
    uint16_t* __restrict__ y = static_cast<uint16_t*>(a.y);
    int t = 0;
    for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      if (!wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag,
                             a.timeout_ns, kSiteEpiAccFull))
        break;
      ptx::tc_fence_after();
      const TileCoord tc = decode_tile(a, tile);
      const long long m = static_cast<long long>(tc.mt) * kBM + row;
      const int n0 = tc.nt * a.BN;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * a.BN);
      const long long ybase = m * a.O + static_cast<long long>(tc.g) * a.Og;
      for (int c = 0; c < a.BN; c += 32) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(taddr + c, r);
        ptx::tmem_ld_wait();
        const int col0 = n0 + c;
        const int nvalid = min(32, a.Og - col0);
        if (m < a.M && nvalid > 0) {
          uint16_t* dst = y + ybase + col0;
          if (nvalid == 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 v;
              v.x = pack2<BF16>(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
              v.y = pack2<BF16>(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
              v.z = pack2<BF16>(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
              v.w = pack2<BF16>(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
              d4[j] = v;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) dst[j] = cvt1<BF16>(__uint_as_float(r[j]));
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&tail->acc_empty[acc]));
    }
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem_base, a.tmem_cols);
}

}  // namespace convfwd
