// conv_tconv.cuh -- the transposed convolution by sub-pixel phases, fed by TMA
// (tcgen05, CTA pairs).
//
// The transposed convolution (see conv_transpose in conv_fwd.h) with filter
// dilation 1 writes output q = s*t + r (per dimension, residue r < s) from the
// taps k with k = (r + p) mod s (mod s): k = k_r + s*j, j < J_r, which read
// input i = t + c_r - j, c_r = (r + p - k_r) / s.  So each phase (r_d, r_h,
// r_w) is a stride-1 convolution of the undilated input over its own tap set,
// with output rows t < T_r = ceil((Q - r) / s), and no product of an inserted
// zero is ever formed.
//
// All phases share one TMA im2col map of x: it walks Tm = max_r T_r pixels per
// dimension from the lower corner L = min_r (c_r - J_r + 1), and phase r's tap
// j is the im2col offset c_r - j - L (>= 0).  Rows of a phase past its own T_r
// are computed over the shared walk and never stored.  B is w itself:
// w [Cin][taps][Cout/G] holds, for one tap, a [ci][co] matrix whose rows are
// 64-channel TMA boxes in the 128-byte swizzle, read as an MN-major operand
// (N = co contiguous; one K step = 16 ci rows = 2 KB; LBO = the next 64-co box).
// A sub-block carries 128 input channels where Cin/G allows (two im2col boxes,
// one 16 KB weight box per 64 output channels), else 64.
//
// CTA pair (cta_group::2): M = 256 phase pixels (128 per CTA, its own im2col
// box), N = BN output channels (each CTA loads the boxes of its BN/2).  A tile
// is (phase, group, channel tile, 256-row block); its K blocks are the phase's
// taps x 64-channel chunks.  The epilogue stores each row of 32 channels with
// 16-byte stores at its output pixel s*t + r (rows of one tile are s pixels
// apart in y, so no tensor store spans them).  A phase with no taps writes
// zeros.
#pragma once

#include <cstdint>

#include "conv_tc.cuh"
#include "ptx.cuh"

namespace convfwd {

constexpr int kTcvMaxStride = 8;
constexpr int kTcvThreads = 192;

struct TconvArgs {
  int N, D, H, W, Cin, Cout, G, Cig, Cog;
  int kD, kH, kW;
  int Qd, Qh, Qw;
  int s[3];
  // per dimension (0 = depth, 1 = height, 2 = width) and residue r < s[dim]
  int ph_k[3][kTcvMaxStride];  // first tap k_r
  int ph_J[3][kTcvMaxStride];  // taps J_r
  int ph_c[3][kTcvMaxStride];  // input offset c_r of tap j = 0
  int ph_T[3][kTcvMaxStride];  // output rows T_r of the phase
  int lower[3];                // im2col lower corner L (the walk's origin)
  int Tm[3];                   // rows the shared walk covers (max_r T_r)
  long long Mph;               // rows per phase: N * Tm[0] * Tm[1] * Tm[2]
  int nphase;                  // s[0] * s[1] * s[2]
  int m_tiles, n_tiles, BN, total_tiles;
  int kc;                      // input channels per sub-block: 128 (when Cig allows) or 64
  int cchunks;                 // Cig / kc
  int kbs, stages;
  uint32_t a_bytes, b_bytes, sub_bytes, stage_bytes;
  uint32_t idesc, tmem_cols;
  int rank5;
  unsigned long long timeout_ns;
  int inject_stall;
  void* y;
};

struct TcvTile {
  int ph, g, nt, mt;
  int r[3];   // residues of the phase
  int J[3];   // its taps per dimension
  int nkb;    // K blocks: J0 * J1 * J2 * cchunks (0: no tap reaches the phase)
};

__device__ __forceinline__ TcvTile tcv_tile(const TconvArgs& a, int t) {
  TcvTile u;
  u.mt = t % a.m_tiles;
  t /= a.m_tiles;
  u.nt = t % a.n_tiles;
  t /= a.n_tiles;
  u.g = t % a.G;
  u.ph = t / a.G;
  u.r[0] = u.ph / (a.s[1] * a.s[2]);
  u.r[1] = (u.ph / a.s[2]) % a.s[1];
  u.r[2] = u.ph % a.s[2];
  u.nkb = a.cchunks;
#pragma unroll
  for (int d = 0; d < 3; ++d) {
    u.J[d] = a.ph_J[d][u.r[d]];
    u.nkb *= u.J[d];
  }
  return u;
}

// Row m of a phase's walk -> (n, td, th, tw).
__device__ __forceinline__ void tcv_row(const TconvArgs& a, long long m, int& n, int& td, int& th, int& tw) {
  tw = static_cast<int>(m % a.Tm[2]);
  long long q = m / a.Tm[2];
  th = static_cast<int>(q % a.Tm[1]);
  q /= a.Tm[1];
  td = static_cast<int>(q % a.Tm[0]);
  n = static_cast<int>(q / a.Tm[0]);
}

// Per-CTA bytes of the f-th pipeline fill of the pair whose first tile is
// `first` (fills of a tile carry min(kbs, remaining K blocks) sub-blocks).
__device__ uint32_t tcv_fill_bytes(const TconvArgs& a, int first, int npairs, long long f) {
  for (int t = first; t < a.total_tiles; t += npairs) {
    const int nkb = tcv_tile(a, t).nkb;
    const long long nf = (nkb + a.kbs - 1) / a.kbs;
    if (f < nf) return static_cast<uint32_t>(min(static_cast<long long>(a.kbs), nkb - f * a.kbs)) * a.sub_bytes;
    f -= nf;
  }
  return 0u;
}

template <bool BF16>
__global__ void __launch_bounds__(kTcvThreads, 1)
    conv_tconv_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                           const TconvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(smem + a.stages * a.stage_bytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int half_bn = a.BN >> 1;

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
    ptx::prefetch_tmap(&tmap_w);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(&tail->tmem_base), a.tmem_cols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // barriers of both CTAs initialised before any remote use
  ptx::tc_fence_after();
  ptx::pdl_allow_next();  // setup done: the next launch may start its own
  ptx::pdl_wait_prev();   // the previous launch's writes are visible from here on
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long fills = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < a.total_tiles; tile += npairs) {
        const TcvTile u = tcv_tile(a, tile);
        if (u.nkb == 0) continue;
        int n, td, th, tw;
        tcv_row(a, static_cast<long long>(u.mt) * 256 + rank * 128, n, td, th, tw);
        const int cw = tw + a.lower[2], chh = th + a.lower[1], cd = td + a.lower[0];
        const int co0 = u.nt * a.BN + static_cast<int>(rank) * half_bn;
        int jd = 0, jh = 0, jw = 0, cc = 0;
        for (int kb = 0; kb < u.nkb; kb += a.kbs) {
          const int nsub = min(a.kbs, u.nkb - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = ptx::smem_u32(&tail->full[stage]);
          if (leader) ptx::mbar_arrive_expect_tx(fb_local, 2u * static_cast<uint32_t>(nsub) * a.sub_bytes);
          const uint32_t fb = ptx::mapa_shared(fb_local, 0);
          for (int j = 0; j < nsub; ++j) {
            const uint32_t sa = ptx::smem_u32(smem + stage * a.stage_bytes + j * a.sub_bytes);
            const uint32_t sb = sa + a.a_bytes;
            // the phase's tap (jd, jh, jw): im2col offsets and the filter tap it multiplies
            const int ow = a.ph_c[2][u.r[2]] - jw - a.lower[2];
            const int oh = a.ph_c[1][u.r[1]] - jh - a.lower[1];
            const int od = a.ph_c[0][u.r[0]] - jd - a.lower[0];
            const int kd = a.ph_k[0][u.r[0]] + a.s[0] * jd;
            const int kh = a.ph_k[1][u.r[1]] + a.s[1] * jh;
            const int kw = a.ph_k[2][u.r[2]] + a.s[2] * jw;
            const int tap = (kd * a.kH + kh) * a.kW + kw;
            const int ci0 = u.g * a.Cig + cc * a.kc;
            // A: one [128 px][64 ch] im2col box per 64 channels of the sub-block
            for (int h = 0; h < a.kc / 64; ++h) {
              if (a.rank5)
                ptx::tma_load_im2col_5d_pair(sa + h * 16384u, &tmap_x, fb, ci0 + h * 64, cw, chh, cd, n,
                                             static_cast<uint16_t>(ow), static_cast<uint16_t>(oh),
                                             static_cast<uint16_t>(od));
              else
                ptx::tma_load_im2col_4d_pair(sa + h * 16384u, &tmap_x, fb, ci0 + h * 64, cw, chh, n,
                                             static_cast<uint16_t>(ow), static_cast<uint16_t>(oh));
            }
            // B: one [kc ci][64 co] box per 64 output channels of this CTA's half
            for (int b = 0; b < half_bn / 64; ++b)
              ptx::tma_load_3d_pair(sb + b * static_cast<uint32_t>(a.kc) * 128u, &tmap_w, fb, co0 + b * 64, tap, ci0);
            if (++cc == a.cchunks) {
              cc = 0;
              if (++jw == u.J[2]) {
                jw = 0;
                if (++jh == u.J[1]) {
                  jh = 0;
                  ++jd;
                }
              }
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
                       [&](long long f) { return tcv_fill_bytes(a, pair, npairs, f); });
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
      // A: K-major im2col rows (K step = 32 bytes within a 64-channel box, the
      // next box 16 KB on); B: MN-major weight boxes (LBO = the next 64-channel
      // box, SBO = 8 ci rows, K step = 16 rows = 2 KB)
      const uint64_t d_a = ptx::smem_desc(ptx::smem_u32(smem), 16, 1024, 2u);
      const uint64_t d_b = ptx::smem_desc(ptx::smem_u32(smem + a.a_bytes), static_cast<uint32_t>(a.kc) * 128u, 1024, 2u);
      const int ksteps = a.kc >> 4;
      const uint64_t sub_off = desc_off(a.sub_bytes), st_off = desc_off(a.stage_bytes);
      for (int tile = pair; ok && tile < a.total_tiles; tile += npairs, ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag, a.timeout_ns,
                          kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const int nkb = tcv_tile(a, tile).nkb;
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        for (int kb = 0; kb < nkb; kb += a.kbs) {
          const int nsub = min(a.kbs, nkb - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t so = static_cast<uint64_t>(stage) * st_off;
          for (int j = 0; j < nsub; ++j) {
            const uint64_t da = d_a + so + static_cast<uint64_t>(j) * sub_off;
            const uint64_t db = d_b + so + static_cast<uint64_t>(j) * sub_off;
            // (unrolled: descriptor offsets are constants)
            if (ksteps == 8) {
#pragma unroll
              for (int k = 0; k < 8; ++k)
                ptx::mma_f16_pair(d_tmem, da + (k >> 2) * 1024 + 2 * (k & 3), db + 128 * k, a.idesc,
                                  (kb + j + k) != 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ptx::mma_f16_pair(d_tmem, da + 2 * k, db + 128 * k, a.idesc, (kb + j + k) != 0 ? 1u : 0u);
            }
          }
          ptx::mma_commit_pair(ptx::smem_u32(&tail->empty[stage]), 3);
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        // (a tile with no K blocks commits at once: its epilogue writes zeros)
        if (ok) ptx::mma_commit_pair(ptx::smem_u32(&tail->acc_full[acc]), 3);
      }
      ptx::mma_commit_pair(ptx::smem_u32(&tail->drain), 1);
      wait_drain(ptx::smem_u32(&tail->drain), 0, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint16_t* __restrict__ y = static_cast<uint16_t*>(a.y);
    int t = 0;
    for (int tile = pair; tile < a.total_tiles; tile += npairs, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      if (!wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                             kSiteEpiAccFull))
        break;
      ptx::tc_fence_after();
      const TcvTile u = tcv_tile(a, tile);
      const long long m = static_cast<long long>(u.mt) * 256 + rank * 128 + row;
      int n, td, th, tw;
      tcv_row(a, m < a.Mph ? m : 0, n, td, th, tw);
      const bool valid = m < a.Mph && td < a.ph_T[0][u.r[0]] && th < a.ph_T[1][u.r[1]] && tw < a.ph_T[2][u.r[2]];
      const int qd = a.s[0] * td + u.r[0], qh = a.s[1] * th + u.r[1], qw = a.s[2] * tw + u.r[2];
      const long long ybase =
          (((static_cast<long long>(n) * a.Qd + qd) * a.Qh + qh) * a.Qw + qw) * a.Cout + u.g * a.Cog + u.nt * a.BN;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
      for (int c = 0; c < a.BN; c += 32) {
        uint32_t r[32];
        if (u.nkb == 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;  // +0.0f
        } else {
          ptx::tmem_ld_32x32b_x32(taddr + c, r);
          ptx::tmem_ld_wait();
        }
        if (valid) {
          uint4* d4 = reinterpret_cast<uint4*>(y + ybase + c);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 v;
            v.x = pack2<BF16>(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
            v.y = pack2<BF16>(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
            v.z = pack2<BF16>(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
            v.w = pack2<BF16>(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
            d4[j] = v;
          }
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
  if (warp == 1) ptx::tmem_dealloc_pair(tmem_base, a.tmem_cols);
}

}  // namespace convfwd
