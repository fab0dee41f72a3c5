// conv_wgrad_tc.cuh -- the weight gradient on the tensor cores (tcgen05, CTA pairs).
//
// dw[o, (tap, c)] = sum over output pixels p of dy[p, o] * X[p, (tap, c)], X the
// im2col matrix of x (the weight gradient of the forward pass; see
// conv_wgrad.cuh).  As a GEMM: M = output channels, N = weight columns
// (tap, channel), K = output pixels.  Both operands arrive exactly as the
// forward kernels load their tiles: dy rows by a 2-D TMA box of [128 pixels]
// [64 output channels], x by a TMA im2col box of [128 pixels][64 channels]
// per tap, both in the 128-byte swizzle.  In the forward pass such a tile is
// a K-major operand (K = channels); here the same bytes are MN-major operands
// (K = pixels, the 64 channels of a row contiguous), which the instruction
// descriptor's transpose bits select: one K step of 16 pixels is two 8-row
// groups (SBO = 1024 bytes apart), the second 64-channel block of a 128-wide
// operand half sits LBO = one box (16 KB) further.
//
// CTA pair (cta_group::2): M = 256 output channels (128 per CTA, their dy
// boxes), N = 256 weight columns (each CTA loads the im2col boxes of its 128).
// Work unit = (group, 256-channel tile, 256-column tile, pixel range); the
// pixel reduction is split into ranges so that the units cover the SMs, each
// unit's fp32 accumulator (TMEM, double-buffered) goes to its range's slice
// of the workspace, and conv_wgrad_reduce_kernel adds the slices in range
// order.  Warp 0 produces (TMA), warp 1 issues MMAs (the leader's lane 0),
// warps 2..5 of both CTAs drain the accumulator to the workspace.
#pragma once

#include <cstdint>

#include "conv_tc.cuh"
#include "ptx.cuh"

namespace convfwd {

struct WgTcArgs {
  int N, D, H, W, C, O, kD, kH, kW;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  int G, Cg, Og, Do, Ho, Wo;
  long long P;           // output pixels N*Do*Ho*Wo
  int ncols;             // taps * Cg (columns of one group's dw)
  int jtiles, otiles;    // 256-column tiles of ncols, 256-channel tiles of Og
  int nsplit;            // ranges of the pixel reduction
  int chunk_sub;         // kWgtBK-pixel sub-blocks per range (a multiple of kbs)
  int total_units;       // G * otiles * jtiles * nsplit
  int kbs, stages;       // sub-blocks per pipeline stage, stages
  uint32_t stage_bytes;  // kbs * kWgtSub
  uint32_t idesc;        // tcgen05 instruction descriptor (both operands MN-major)
  int rank5;
  unsigned long long timeout_ns;
  int inject_stall;
  float* part;           // [nsplit][O][ncols] fp32 partial sums
};

constexpr int kWgtBK = 128;                   // pixels per sub-block (K)
constexpr uint32_t kWgtBox = kWgtBK * 128;    // one [128 px][64 ch] box, 128-byte rows
constexpr uint32_t kWgtSub = 4 * kWgtBox;     // per CTA: two dy boxes (A) + two im2col boxes (B)
constexpr int kWgtThreads = 192;
constexpr uint32_t kWgtTmemCols = 512;        // two 256-column fp32 accumulators

struct WgUnit {
  int g, ot, jt, split;
};

__device__ __forceinline__ WgUnit wgt_unit(const WgTcArgs& a, int u) {
  WgUnit r;
  r.split = u % a.nsplit;
  u /= a.nsplit;
  r.jt = u % a.jtiles;
  u /= a.jtiles;
  r.ot = u % a.otiles;
  r.g = u / a.otiles;
  return r;
}

template <bool BF16>
__global__ void __launch_bounds__(kWgtThreads, 1)
    conv_wgrad_tc_pair_kernel(const __grid_constant__ CUtensorMap tmap_x,
                              const __grid_constant__ CUtensorMap tmap_dy, const WgTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(smem + a.stages * a.stage_bytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->full[s]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->empty[s]), 1u);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&tail->acc_full[b]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->acc_empty[b]), 8u);  // 4 epilogue warps x 2 CTAs
    }
    ptx::mbar_init(ptx::smem_u32(&tail->drain), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->stall), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->peer_done), 1u);
    tail->abort_flag = 0;
    tail->peer_fills = 0;
    ptx::fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_dy);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(&tail->tmem_base), kWgtTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // barriers of both CTAs initialised before any remote use
  ptx::tc_fence_after();
  // (no early trigger: the ordered sum that follows this kernel would wait
  // beside it on every SM; it starts as these CTAs exit)
  ptx::pdl_wait_prev();   // the previous launch's writes are visible from here on
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const long long spp = static_cast<long long>(a.Do) * a.Ho * a.Wo;  // output pixels per image

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long fills = 0;
      bool ok = true;
      for (int u = pair; ok && u < a.total_units; u += npairs) {
        const WgUnit w = wgt_unit(a, u);
        const int o_base = w.g * a.Og + w.ot * 256 + static_cast<int>(rank) * 128;  // dy channel
        // this CTA's two 64-column blocks: tap and channel of each (columns past
        // the group's last tap, in a partial last tile, load tap 0 and are never stored)
        int cb[2], offw[2], offh[2], offd[2];
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int j = w.jt * 256 + static_cast<int>(rank) * 128 + b * 64;
          const int tap = j < a.ncols ? j / a.Cg : 0;
          cb[b] = w.g * a.Cg + (j < a.ncols ? j - tap * a.Cg : 0);
          const int kw = tap % a.kW, kh = (tap / a.kW) % a.kH, kd = tap / (a.kW * a.kH);
          offw[b] = kw * a.dw;
          offh[b] = kh * a.dh;
          offd[b] = kd * a.dd;
        }
        const long long sb0 = static_cast<long long>(w.split) * a.chunk_sub;
        for (int f = 0; f < a.chunk_sub; f += a.kbs) {
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = ptx::smem_u32(&tail->full[stage]);
          if (leader) ptx::mbar_arrive_expect_tx(fb_local, 2u * static_cast<uint32_t>(a.kbs) * kWgtSub);
          const uint32_t fb = ptx::mapa_shared(fb_local, 0);
          for (int j = 0; j < a.kbs; ++j) {
            // pixels p0 .. p0+kWgtBK-1 of the range; past the last pixel every box reads zeros
            const long long p0 = (sb0 + f + j) * kWgtBK;
            const long long n = p0 / spp;
            long long r = p0 - n * spp;
            const int od = static_cast<int>(r / (static_cast<long long>(a.Ho) * a.Wo));
            r -= static_cast<long long>(od) * a.Ho * a.Wo;
            const int oh = static_cast<int>(r / a.Wo);
            const int ow = static_cast<int>(r - static_cast<long long>(oh) * a.Wo);
            const int cw = ow * a.sw - a.pw, chh = oh * a.sh - a.ph, cd = od * a.sd - a.pd;
            const uint32_t base = ptx::smem_u32(smem + stage * a.stage_bytes + j * kWgtSub);
            const int pr = static_cast<int>(p0);
            ptx::tma_load_2d_pair(base, &tmap_dy, fb, o_base, pr);
            ptx::tma_load_2d_pair(base + kWgtBox, &tmap_dy, fb, o_base + 64, pr);
            const int ni = static_cast<int>(n);
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              const uint32_t dst = base + (2 + b) * kWgtBox;
              if (a.rank5)
                ptx::tma_load_im2col_5d_pair(dst, &tmap_x, fb, cb[b], cw, chh, cd, ni, static_cast<uint16_t>(offw[b]),
                                             static_cast<uint16_t>(offh[b]), static_cast<uint16_t>(offd[b]));
              else
                ptx::tma_load_im2col_4d_pair(dst, &tmap_x, fb, cb[b], cw, chh, ni, static_cast<uint16_t>(offw[b]),
                                             static_cast<uint16_t>(offh[b]));
            }
          }
          ++fills;
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      pair_settle_ring(tail, a.stages, leader, fills, a.timeout_ns,
                       [&](long long) { return static_cast<uint32_t>(a.kbs) * kWgtSub; });
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int t = 0;
      if (a.inject_stall)
        ok = wait_bounded(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected);
      // MN-major operands, 128-byte swizzle: LBO = the second 64-wide block, SBO = 8 pixel rows
      const uint64_t d_ring = ptx::smem_desc(ptx::smem_u32(smem), kWgtBox, 1024, 2u);
      const uint64_t b_off = desc_off(2 * kWgtBox), sub_off = desc_off(kWgtSub), st_off = desc_off(a.stage_bytes);
      const uint64_t k_off = desc_off(16 * 128);  // one K step: 16 pixel rows of 128 bytes
      for (int u = pair; ok && u < a.total_units; u += npairs, ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag, a.timeout_ns,
                          kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        uint32_t accum = 0u;
        for (int f = 0; f < a.chunk_sub; f += a.kbs) {
          if (!wait_bounded(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          uint64_t da = d_ring + static_cast<uint64_t>(stage) * st_off;
          for (int j = 0; j < a.kbs; ++j) {
#pragma unroll
            for (int k = 0; k < kWgtBK / 16; ++k) {
              ptx::mma_f16_pair(d_tmem, da + k * k_off, da + b_off + k * k_off, a.idesc, accum);
              accum = 1u;
            }
            da += sub_off;
          }
          ptx::mma_commit_pair(ptx::smem_u32(&tail->empty[stage]), 3);
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) ptx::mma_commit_pair(ptx::smem_u32(&tail->acc_full[acc]), 3);
      }
      ptx::mma_commit_pair(ptx::smem_u32(&tail->drain), 1);
      wait_drain(ptx::smem_u32(&tail->drain), 0, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int row = q * 32 + lane;  // output channel within this CTA's 128
    int t = 0;
    for (int u = pair; u < a.total_units; u += npairs, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      if (!wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                             kSiteEpiAccFull))
        break;
      ptx::tc_fence_after();
      const WgUnit w = wgt_unit(a, u);
      const int o = w.g * a.Og + w.ot * 256 + static_cast<int>(rank) * 128 + row;
      float* __restrict__ dst = a.part + (static_cast<long long>(w.split) * a.O + o) * a.ncols + w.jt * 256;
      const int ncols = min(256, a.ncols - w.jt * 256);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * 256);
      for (int c = 0; c < ncols; c += 32) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(taddr + c, r);
        ptx::tmem_ld_wait();
        if (c + 32 <= ncols) {
          float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c + i < ncols) dst[c + i] = __uint_as_float(r[i]);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(&tail->acc_empty[acc]), 0));
    }
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the leader's MMAs (which read this CTA's smem) are complete
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc_pair(tmem_base, kWgtTmemCols);
}

}  // namespace convfwd
