// conv_phase.cuh -- tcgen05 implicit-GEMM convolution forward for 2-D layers
// with few input channels (the C = 3 stem of the "Convolutions" tutorial,
// sections 3 and 5), whose pixels are too narrow for a TMA im2col load.
//
// Phase packing.  With the input row (n, ih) flattened to R[e] = x[n, ih, e/C,
// e%C], output pixel ow reads, for filter row kh, the kW*C consecutive
// elements starting at (ow*sw - pw)*C (width dilation 1).  Pixels ow and ow+1
// start sw*C elements apart, which for C = 3 is not a 16-byte step, but P
// pixels in a row start P*sw*C elements apart, a multiple of 8 elements for
// the smallest suitable P (4 for the stem: 24 elements, 48 bytes).  So one
// GEMM row q stands for P output pixels ow = P*q + i, i < P:
//   A[q, k]        = R[P*sw*C*q - al + k],          k < Kw   (al = pw*C rounded up to 8)
//   B[(i, o), k]   = w[o, kh, (k - off_i) / C, (k - off_i) % C]  if 0 <= k - off_i < kW*C, else 0,
//                    off_i = al - pw*C + i*sw*C
//   D[q, (i, o)]  += sum_k A[q, k] B[(i, o), k]      over the kH filter rows
// and D[q, (i, o)] = y[n, oh, P*q + i, o]: row q of D is P*O consecutive
// elements of y.  N = P*O (256 for the stem); Kw/16 MMA K steps per filter
// row (3 for the stem: a 48-element window holds all four 21-element pixel
// windows).  The zeros of B cost tensor cycles (48 / 21 for the stem), but the
// layer is bound by its output writes.
//
// A rows are 16-byte aligned windows of an input row, so TMA loads them
// straight into the 128-byte-swizzle K-major layout (64-element rows, of
// which the MMAs read the first Kw): one 5-D box of a tensor map whose "row"
// dimension steps P*sw*C elements (overlapping windows) brings the rows whose
// window lies inside the input row, and a plain row map (zero-filled outside
// the row) brings the few edge rows at each end, whose windows reach into the
// left or right padding.  Rows of a CTA's tile are (output row r < ph_rows,
// window q); input rows ih = oh*sh - ph + kh*dh are addressed as (ih % sh,
// ih / sh) so that the tile's output rows are one box dimension; rows outside
// the image read zero.
//
// CTA pairs (cta_group::2): the pair's MMA is M = 256 (each CTA's 128 GEMM
// rows: ph_rows output rows each) x N; each CTA holds half of B's N rows,
// built once in shared memory (by warps 1..5, from a bulk copy of w, while
// the producer already loads the first windows) and kept resident for all
// tiles.  The epilogue reorders each CTA's accumulator rows (interior windows
// first, then the edge windows) into output order, ph_gcols columns at a
// time, in a swizzled staging tile of 128- (or 64-) byte rows, and stores it
// with a 4-D TMA store on y viewed as [N, Ho, Wo/P, P*O], which clips rows
// past Ho.  (Narrower store rows cost the TMA unit as much per row.)
//
// Warp roles (192 threads per CTA, one CTA per SM, static tile list): warp 0
// TMA producer (both CTAs; loads complete on the leader's barriers), warp 1
// TMEM allocator and, in the leader, MMA issuer, warps 2..5 epilogue.  Waits
// are bounded as in the other tcgen05 kernels.
#pragma once

#include "conv_tct.cuh"

namespace convfwd {

constexpr int kPhThreads = 192;
constexpr int kPhWin = 64;                          // elements of a loaded window row (128 bytes)
constexpr uint32_t kPhAStage = kBM * kPhWin * 2;    // one filter row's A tile: 128 rows x 128 bytes

template <bool BF16>
__global__ void __launch_bounds__(kPhThreads, 1)
    conv_fwd_tc_phase_kernel(const __grid_constant__ CUtensorMap tmap_in, const __grid_constant__ CUtensorMap tmap_edge,
                             const __grid_constant__ CUtensorMap tmap_y, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* aring = smem;                                                   // stages x one filter row
  uint8_t* bres = aring + static_cast<size_t>(a.stages) * kPhAStage;       // kH blocks of BN/2 rows x 128 B
  uint8_t* stage_y = bres + static_cast<size_t>(a.kH) * a.ph_bblk;         // 2 staging tiles (first: w)
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(stage_y + 2 * a.ph_epi_bytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int BN = a.BN;       // P * O
  const int hb = BN / 2;     // B rows held by this CTA: rank*hb .. rank*hb + hb - 1

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
    ptx::mbar_init(ptx::smem_u32(&tail->bres), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->bready), 2u);  // one arrival per CTA of the pair
    ptx::mbar_init(ptx::smem_u32(&tail->peer_done), 1u);
    tail->abort_flag = 0;
    tail->peer_fills = 0;
    ptx::fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    ptx::prefetch_tmap(&tmap_in);
    ptx::prefetch_tmap(&tmap_edge);
    ptx::prefetch_tmap(&tmap_y);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_u32(&tail->tmem_base), a.tmem_cols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  ptx::pdl_allow_next();  // setup done: the next launch may start its own
  ptx::pdl_wait_prev();   // the previous launch's writes are visible from here on
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;

  // ---------------------------------------------------------------- resident B
  // w arrives by one bulk copy into the staging tiles (unused until the first
  // accumulator is ready, which needs B); its last w_bytes % 16 bytes by plain
  // loads.  Warps 1..5 build this CTA's half of B from it; warp 0 starts
  // loading windows meanwhile.  The leader's MMA thread waits on `bready`.
  if (warp != 0) {
    const uint16_t* w_s = reinterpret_cast<const uint16_t*>(stage_y);
    const uint32_t wb16 = a.ph_wbytes & ~15u;
    const int btid = threadIdx.x - 32;
    constexpr int kBuilders = kPhThreads - 32;  // warps 1..5: all of them arrive on named barrier 2
    static_assert(kBuilders == 160, "the B builders are exactly warps 1..5");
    bool ok = true;
    if (btid == 0) {
      if (wb16 > 0) {
        ptx::mbar_arrive_expect_tx(ptx::smem_u32(&tail->bres), wb16);
        ptx::bulk_load(ptx::smem_u32(stage_y), a.w, wb16, ptx::smem_u32(&tail->bres));
      }
      const uint16_t* wg = static_cast<const uint16_t*>(a.w);
      uint16_t* wt = reinterpret_cast<uint16_t*>(stage_y);
      for (uint32_t e = wb16 / 2; e < a.ph_wbytes / 2; ++e) wt[e] = wg[e];
    }
    if (wb16 > 0) {
      ok = wait_bounded(ptx::smem_u32(&tail->bres), 0u, abort_flag, a.timeout_ns, kSiteMmaFull);
      // the copy must have landed before this CTA can exit, whatever happened
      if (!ok && btid == 0) wait_drain(ptx::smem_u32(&tail->bres), 0u, a.timeout_ns);
    }
    named_bar_sync(2, kBuilders);  // the plain-loaded tail of w is visible
    if (ok) {
      // B rows eight per warp step, phase-major: for each filter row kh and
      // phase i (window offset off_i) this CTA holds, lane l forms word l
      // (elements 2l, 2l+1) of the 64-element rows of output channels o0..o0+7
      // -- loads from clamped indices, all 16 issued before the step's stores,
      // then masked outside the filter row -- and the warp stores each
      // 128-byte row in the 128-byte swizzle (16-byte chunk XOR row % 8).
      const int KWC = a.kW * a.C;
      const int taps_row = a.kH * KWC;  // elements of one output channel's weights
      const int bwarp = btid >> 5;
      constexpr int kBuilderWarps = kBuilders / 32;
      const uint32_t ws_addr = ptx::smem_u32(w_s);
      const uint32_t b_addr = ptx::smem_u32(bres);
      const int r0 = static_cast<int>(rank) * hb;  // first B row of this CTA
      const int i_begin = r0 / a.O, i_end = (r0 + hb + a.O - 1) / a.O;
      for (int kh = 0; kh < a.kH; ++kh) {
        for (int i = i_begin; i < i_end; ++i) {
          const int off = a.ph_align - a.pw * a.C + i * a.sw * a.C;
          const int ja = 2 * lane - off, jb = ja + 1;
          const uint32_t ma = static_cast<unsigned>(ja) < static_cast<unsigned>(KWC) ? 0xffffu : 0u;
          const uint32_t mb = static_cast<unsigned>(jb) < static_cast<unsigned>(KWC) ? 0xffffu : 0u;
          // element j = kw*C + c of the filter row; with flip it reads filter row
          // kH-1-kh (below) and, within it, kw mirrored: (kW-1-kw)*C + c
          const auto src_elem = [&](int j) {
            const int jc = min(max(j, 0), KWC - 1);
            return a.flip ? (a.kW - 1 - jc / a.C) * a.C + jc % a.C : jc;
          };
          const uint32_t ca = 2u * static_cast<uint32_t>(src_elem(ja));
          const uint32_t cb = 2u * static_cast<uint32_t>(src_elem(jb));
          const int kh_src = a.flip ? a.kH - 1 - kh : kh;
          const int o_begin = max(0, r0 - i * a.O), o_end = min(a.O, r0 + hb - i * a.O);
          const int lrb = i * a.O - r0;  // this CTA's B row of (i, o = 0)
          const uint32_t blk = b_addr + static_cast<uint32_t>(kh) * a.ph_bblk + ((lane & 3) << 2);
          for (int o0 = o_begin + 8 * bwarp; o0 < o_end; o0 += 8 * kBuilderWarps) {
            uint32_t ha[8], hv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int o = min(o0 + u, o_end - 1);
              const uint32_t base = ws_addr + 2u * static_cast<uint32_t>(o * taps_row + kh_src * KWC);
              ha[u] = lds16(base + ca);
              hv[u] = lds16(base + cb);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              if (o0 + u < o_end) {
                const int lr = lrb + o0 + u;
                const uint32_t v = (ha[u] & ma) | ((hv[u] & mb) << 16);
                asm volatile("st.shared.b32 [%0], %1;"
                             ::"r"(blk + static_cast<uint32_t>(lr) * 128u + (((lane >> 2) ^ (lr & 7)) << 4)), "r"(v)
                             : "memory");
              }
            }
          }
        }
      }
      ptx::fence_proxy_async_smem();  // B (generic-proxy stores) before the tensor core reads it
    }
    named_bar_sync(2, kBuilders);
    // the leader's MMAs read both CTAs' halves: each CTA reports to the leader
    // (nothing arrives after a failed copy; the MMA thread's wait then runs out)
    if (btid == 0 && ok) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(&tail->bready), 0));
  }

  const int R = a.ph_rows;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long fills = 0;
      bool pok = !*abort_flag;  // (no loads at all after a failed copy of w)
      const int nedge = a.ph_nleft + a.ph_nright;
      const uint32_t bytes = static_cast<uint32_t>((R * a.ph_qint + nedge * R) * kPhWin * 2);
      const int pitch = a.ph_P * a.sw * a.C;  // elements between consecutive windows
      for (int tile = static_cast<int>(blockIdx.x >> 1); pok && tile < a.total_tiles;
           tile += static_cast<int>(gridDim.x >> 1)) {
        const int n = tile / a.tiles_h;
        const int oh0 = (tile - n * a.tiles_h) * 2 * R + static_cast<int>(rank) * R;  // this CTA's rows
        for (int kh = 0; kh < a.kH; ++kh) {
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            pok = false;
            break;
          }
          const uint32_t fb = ptx::smem_u32(&tail->full[stage]);
          if (leader) ptx::mbar_arrive_expect_tx(fb, 2u * bytes);
          const uint32_t fb_l = ptx::mapa_shared(fb, 0);
          // input row ih = oh*sh + dy as (parity, ih / sh); exact division below
          const int dy = kh * a.dh - a.ph;
          const int par = ((dy % a.sh) + a.sh) % a.sh;
          const int hp0 = oh0 + (dy - par) / a.sh;
          const uint32_t dst = ptx::smem_u32(aring + static_cast<size_t>(stage) * kPhAStage);
          ptx::tma_load_5d_pair(dst, &tmap_in, fb_l, 0, 0, par, hp0, n);
          for (int j = 0; j < nedge; ++j) {
            const int q = j < a.ph_nleft ? j : a.ph_qtot - a.ph_nright + (j - a.ph_nleft);
            ptx::tma_load_4d_pair(dst + static_cast<uint32_t>((a.ph_erow0 + 8 * j) * kPhWin * 2), &tmap_edge,
                                  fb_l, pitch * q - a.ph_align, par, hp0, n);
          }
          ++fills;
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // a pair's loads all complete on the leader's barriers: the two producers
      // settle every fill either issued (each carries `bytes` per CTA)
      pair_settle_ring(tail, a.stages, leader, fills, a.timeout_ns, [&](long long) { return bytes; });
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (the leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool mok = !*abort_flag;
      int t = 0;
      if (mok && a.inject_stall)
        mok = wait_bounded(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected);
      if (mok) mok = wait_bounded(ptx::smem_u32(&tail->bready), 0u, abort_flag, a.timeout_ns, kSiteMmaFull);
      ptx::tc_fence_after();
      const uint64_t d_a = ptx::smem_desc(ptx::smem_u32(aring), 16, 1024, 2u);  // 128-byte swizzle
      const uint64_t d_b = ptx::smem_desc(ptx::smem_u32(bres), 16, 1024, 2u);
      const uint64_t st_off = desc_off(kPhAStage), bblk = desc_off(a.ph_bblk);
      for (int tile = static_cast<int>(blockIdx.x >> 1); mok && tile < a.total_tiles;
           tile += static_cast<int>(gridDim.x >> 1), ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag, a.timeout_ns,
                          kSiteMmaAccEmpty)) {
          mok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kh = 0; kh < a.kH; ++kh) {
          if (!wait_bounded(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            mok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t da = d_a + static_cast<uint64_t>(stage) * st_off;
          const uint64_t db = d_b + static_cast<uint64_t>(kh) * bblk;
          // K steps of 16 elements are 32 bytes along the swizzled rows
          mma_sub<true>(a.ph_ks, d_tmem, da, db, a.idesc, kh != 0 ? 1u : 0u);
          ptx::mma_commit_pair(ptx::smem_u32(&tail->empty[stage]), 3);
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (mok) ptx::mma_commit_pair(ptx::smem_u32(&tail->acc_full[acc]), 3);
      }
      // every MMA this thread issued has completed once `drain` fires
      ptx::mma_commit_pair(ptx::smem_u32(&tail->drain), 1);
      wait_drain(ptx::smem_u32(&tail->drain), 0, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Accumulator row m = 32*(warp % 4) + lane holds the window of (output
    // row r, GEMM row q): interior windows are rows r*qint + (q - nleft),
    // edge window j (left ones first) rows erow0 + 8j + r.  Its 32 columns
    // per step go to staging position r*qtot + q, 64 bytes each.
    const int qd = warp & 3;
    const int m = qd * 32 + lane;
    int pos = -1;
    if (m < R * a.ph_qint) {
      const int r = m / a.ph_qint;
      pos = r * a.ph_qtot + a.ph_nleft + (m - r * a.ph_qint);
    } else if (m >= a.ph_erow0) {
      const int j = (m - a.ph_erow0) >> 3, r = (m - a.ph_erow0) & 7;
      if (j < a.ph_nleft + a.ph_nright && r < R)
        pos = r * a.ph_qtot + (j < a.ph_nleft ? j : a.ph_qtot - a.ph_nright + (j - a.ph_nleft));
    }
    const bool store_thread = warp == 2 && lane == 0;
    const int G = a.ph_gcols;               // columns per store: 64 (128-byte rows) or 32 (64-byte)
    const int row_bytes = 2 * G;
    const int sw_mask = G == 64 ? 7 : 3;    // 16-byte chunk XOR pattern of the row's swizzle
    const int sw_shift = G == 64 ? 0 : 1;
    int t = 0, seq = 0;
    for (int tile = static_cast<int>(blockIdx.x >> 1); tile < a.total_tiles;
         tile += static_cast<int>(gridDim.x >> 1), ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      bool eok = !*abort_flag && wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag,
                                                  a.timeout_ns, kSiteEpiAccFull);
      // the four warps agree before any of them enters the named barriers below
      eok = named_bar_and(1, 128, eok);
      if (!eok) break;
      ptx::tc_fence_after();
      const int n = tile / a.tiles_h;
      const int oh0 = (tile - n * a.tiles_h) * 2 * R + static_cast<int>(rank) * R;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const bool live = oh0 < a.Ho;  // this CTA's rows of the last pair tile may lie past the output
      for (int g = 0; g < BN; g += G) {
        uint8_t* buf = stage_y + (seq & 1) * a.ph_epi_bytes;
        if (live) {
          // the store issued two groups ago read this buffer; it must be done
          if (store_thread) ptx::bulk_wait_group_read<1>();
          named_bar_sync(1, 128);
        }
        // both 32-column halves of a 64-column group in flight before one wait
        uint32_t r[2][32];
        ptx::tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(g), r[0]);
        if (G == 64) ptx::tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(g + 32), r[1]);
        ptx::tmem_ld_wait();
        if (live && pos >= 0) {
          uint8_t* rowp = buf + pos * row_bytes;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h * 32 >= G) break;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 v;
              v.x = pack2<BF16>(__uint_as_float(r[h][8 * j + 0]), __uint_as_float(r[h][8 * j + 1]));
              v.y = pack2<BF16>(__uint_as_float(r[h][8 * j + 2]), __uint_as_float(r[h][8 * j + 3]));
              v.z = pack2<BF16>(__uint_as_float(r[h][8 * j + 4]), __uint_as_float(r[h][8 * j + 5]));
              v.w = pack2<BF16>(__uint_as_float(r[h][8 * j + 6]), __uint_as_float(r[h][8 * j + 7]));
              const int chunk = 4 * h + j;  // 16-byte chunk of the staging row
              *reinterpret_cast<uint4*>(rowp + ((chunk ^ ((pos >> sw_shift) & sw_mask)) << 4)) = v;
            }
          }
        }
        if (live) {
          ptx::fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (store_thread) {
            ptx::tma_store_4d(&tmap_y, ptx::smem_u32(buf), g, 0, oh0, n);
            ptx::bulk_commit_group();
          }
          ++seq;
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      // the pair's accumulator buffer is reused once both CTAs' epilogues are done
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(&tail->acc_empty[acc]), 0));
    }
    // every store has finished (reading shared memory and writing y) before exit
    if (store_thread) ptx::bulk_wait_group<0>();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the leader's MMAs (which read this CTA's smem) are complete
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc_pair(tmem_base, a.tmem_cols);
}

}  // namespace convfwd
