// conv_halo_t.cuh -- tcgen05 implicit-GEMM convolution forward, transposed
// orientation with input-halo reuse (stride 1, C/G % 64 == 0, O/G % 128 == 0).
//
// The product is issued as y^T[o, m] = sum_k W[o, k] X[m, k] (see
// conv_tct.cuh): MMA M = 128 output channels (A = a weight tile), N = 256
// output pixels (B = patch rows).  The pixels are a block of tile_h x 8
// output pixels (h x w, tile_h <= 32) of one (n, od) plane, and B is not
// loaded per tap:
// for each 64-channel chunk, depth tap kd and width tap kw, ONE tiled TMA box
// brings the input column strip the block needs -- (tile_h + dh*(kH-1)) rows x 8
// columns (shifted by kw*dw) x 64 channels, zero-filled outside the image --
// and every height tap kh reads a view of it that starts kh*dh rows down.
// Pixel j = r*8 + c of the block reads strip pixel (r + kh*dh, c); the strip is
// exactly 8 pixels wide, so each group of 8 B rows is one strip row (1024
// bytes, one whole 128B-swizzle atom) and every view is a standard K-major
// operand: 1024-byte aligned, stride (SBO) 1024.  (Views that start at other
// rows are valid operands too, but on B200 the MMA reads them markedly slower.)
//
// Compared with per-tap im2col loads this fetches each input pixel once per
// (chunk, kd, kw) instead of kH*kW times per (chunk, kd): per 64-deep K block
// 16 KB of weights plus strip/kH instead of 16 KB plus 32 KB of patch rows.
//
// Epilogue: the accumulator holds [128 channels][8 * tile_h pixels]; 32 columns are
// 4 output rows x 8 output columns.  Four warps transpose each such chunk into
// a [4][8][128] staging tile and one thread stores it with a 4-D / 5-D TMA
// tensor store on y viewed as [N, (Do,) Ho, Wo, O], which clips the rows and
// columns of the block that fall outside the output.
#pragma once

#include "conv_halo.cuh"
#include "conv_tct.cuh"

namespace convfwd {

// Output block: tile_h (4 .. 32, a multiple of 4, chosen by the host to fit Ho)
// x 8 pixels, so MMA N = 8 * tile_h <= 256.  The two accumulators sit 256
// tensor-memory columns apart whatever N is.
constexpr int kHTBlockHMax = 32, kHTBlockW = 8;
constexpr uint32_t kHTAccStride = 256;
constexpr uint32_t kTEpiWarpBytes = kTEpiBytes / 4;

struct HaloTTile {
  int g, n, od, h0, w0, ot;
};

// Tile -> (group, image, output depth, block origin, 128-channel output tile).
// Output-channel tiles vary fastest so that CTAs working at the same time
// share the input block through L2.
__device__ __forceinline__ HaloTTile decode_halo_t_tile(const TcArgs& a, int tile) {
  HaloTTile t;
  t.ot = tile % a.n_tiles;
  int q = tile / a.n_tiles;
  const int tw = q % a.tiles_w;
  q /= a.tiles_w;
  const int th = q % a.tiles_h;
  q /= a.tiles_h;
  const int plane = q % (a.N * a.Do);
  t.g = q / (a.N * a.Do);
  t.od = plane % a.Do;
  t.n = plane / a.Do;
  t.h0 = th * a.tile_h;
  t.w0 = tw * a.tile_w;
  return t;
}

template <bool BF16, bool PAIR>
__global__ void __launch_bounds__(kTThreads, 1)
    conv_fwd_tc_halo_t_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                              const __grid_constant__ CUtensorMap tmap_y, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* halo = smem;                                              // a_slots x halo_slot_bytes
  uint8_t* bring = smem + a.a_slots * a.halo_slot_bytes;             // stages x (kbs weight tiles)
  uint8_t* stage_y = bring + static_cast<size_t>(a.stages) * a.stage_bytes;  // epi_bufs staging tiles
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(stage_y + a.epi_bufs * kTEpiBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const uint32_t mult = PAIR ? 2u : 1u;  // CTAs whose loads complete on the leader's barriers

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->full[s]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->empty[s]), 1u);
    }
    for (int s = 0; s < a.a_slots; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->afull[s]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->aempty[s]), 1u);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&tail->acc_full[b]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->acc_empty[b]), PAIR ? 8u : 4u);
    }
    ptx::mbar_init(ptx::smem_u32(&tail->drain), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->stall), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->peer_done), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->peer_done_a), 1u);
    tail->abort_flag = 0;
    tail->peer_fills = 0;
    tail->peer_fills_a = 0;
    ptx::fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_y);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      ptx::tmem_alloc_pair(ptx::smem_u32(&tail->tmem_base), a.tmem_cols);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(ptx::smem_u32(&tail->tmem_base), a.tmem_cols);
      ptx::tmem_relinquish();
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) ptx::cluster_sync();
  ptx::tc_fence_after();
  ptx::pdl_allow_next();  // setup done: the next launch may start its own
  ptx::pdl_wait_prev();   // the previous launch's writes are visible from here on
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;
  const int taps_hw = a.kH * a.kW;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nunits = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int mo = a.mo;                      // output channels per CTA (MMA M per CTA: 64 or 128)
  const int o_tile = PAIR ? 2 * mo : mo;    // output channels per tile
  const int BP = a.BN;  // 8 * tile_h output pixels per tile

  // K blocks of a tile in issue order: q = ((cc * kD + kd) * kW + kw) * kH + kh.
  // A pipeline stage holds up to kbs consecutive K blocks (weight tiles); each
  // (cc, kd, kw) group has one strip in its own ring of a_slots slots.
  const int Q = a.cchunks * a.kD * taps_hw;
  if (warp == 0) {
    // ------------------------------------------------------------ producers
    // Two threads, each running ahead on its own ring: lane 0 streams the
    // weight tiles, lane 1 the input strips.  Each arms a barrier only right
    // before issuing every load it covers, so a wait that gives up never
    // leaves a barrier expecting bytes that were not requested.
    if (lane == 0) {
      int bst = 0;
      uint32_t bph = 0;
      long long bfills = 0;
      bool ok = true;
      // resident weights (one output-channel tile, one group): the first
      // tile's single fill of stage 0 serves every tile
      const int tile_end = a.w_resident ? min(a.total_tiles, unit + 1) : a.total_tiles;
      for (int tile = unit; ok && tile < tile_end; tile += nunits) {
        const HaloTTile ht = decode_halo_t_tile(a, tile);
        const int orow = ht.g * a.Og + ht.ot * o_tile + static_cast<int>(rank) * mo;
        int kh = 0, kw = 0, kd = 0, cc = 0;  // tap of the next K block (kh fastest, then kw, kd, cc)
        for (int q0 = 0; ok && q0 < Q; q0 += a.kbs) {
          const int nsub = min(a.kbs, Q - q0);
          if (!wait_bounded(ptx::smem_u32(&tail->empty[bst]), bph ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = ptx::smem_u32(&tail->full[bst]);
          if (leader) ptx::mbar_arrive_expect_tx(fb, mult * static_cast<uint32_t>(nsub) * a.b_bytes);
          const uint32_t fb_l = PAIR ? ptx::mapa_shared(fb, 0) : fb;
          for (int j = 0; j < nsub; ++j) {
            const uint32_t sb = ptx::smem_u32(bring + bst * a.stage_bytes + j * a.b_bytes);
            const int tap = (kd * a.kH + kh) * a.kW + kw;  // weight layout (kd, kh, kw)
            if constexpr (PAIR) ptx::tma_load_2d_pair(sb, &tmap_w, fb_l, wtap(a, tap) * a.Cg + cc * a.kc, orow);
            else ptx::tma_load_2d(sb, &tmap_w, fb, wtap(a, tap) * a.Cg + cc * a.kc, orow);
            if (++kh == a.kH) {
              kh = 0;
              if (++kw == a.kW) {
                kw = 0;
                if (++kd == a.kD) {
                  kd = 0;
                  ++cc;
                }
              }
            }
          }
          ++bfills;
          if (++bst == a.stages) {
            bst = 0;
            bph ^= 1u;
          }
        }
      }
      if constexpr (PAIR) {
        // both CTAs' loads complete on the leader's barriers: the two producers
        // settle every fill either issued (the resident fill included)
        const int fpt = (Q + a.kbs - 1) / a.kbs;
        pair_settle_ring(tail, a.stages, leader, bfills, a.timeout_ns, [&](long long k) {
          return static_cast<uint32_t>(min(a.kbs, Q - static_cast<int>(k % fpt) * a.kbs)) * a.b_bytes;
        });
      } else if (a.w_resident && ok && bfills > 0) {
        // the MMA thread may give up before it waits on the resident fill:
        // the loads must have landed before this CTA can exit
        wait_drain(ptx::smem_u32(&tail->full[0]), 0u, a.timeout_ns);
      } else if (!ok) {
        for (int s = 0; s < a.stages; ++s) {
          const long long arms = bfills / a.stages + (s < bfills % a.stages ? 1 : 0);
          if (arms > 0) wait_drain(ptx::smem_u32(&tail->full[s]), static_cast<uint32_t>((arms - 1) & 1), a.timeout_ns);
        }
      }
    } else if (lane == 1) {
      int ast = 0;
      uint32_t aph = 0;
      long long afills = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < a.total_tiles; tile += nunits) {
        const HaloTTile ht = decode_halo_t_tile(a, tile);
        for (int cc = 0; ok && cc < a.cchunks; ++cc)
          for (int kd = 0; ok && kd < a.kD; ++kd)
            for (int kw = 0; kw < a.kW; ++kw) {
              if (!wait_bounded(ptx::smem_u32(&tail->aempty[ast]), aph ^ 1u, abort_flag, a.timeout_ns,
                                kSiteProducerEmpty)) {
                ok = false;
                break;
              }
              const uint32_t afb = ptx::smem_u32(&tail->afull[ast]);
              if (leader) ptx::mbar_arrive_expect_tx(afb, mult * a.halo_bytes);
              const uint32_t afb_l = PAIR ? ptx::mapa_shared(afb, 0) : afb;
              const uint32_t dst = ptx::smem_u32(halo + ast * a.halo_slot_bytes);
              const int c0 = ht.g * a.Cg + cc * a.kc;
              // a pair splits the block's rows: each CTA loads the strip of its half
              const int wc = ht.w0 - a.pw + kw * a.dw;
              const int hc = ht.h0 + static_cast<int>(rank) * (a.tile_h / 2) - a.ph;
              const int dc = ht.od - a.pd + kd * a.dd;
              if constexpr (PAIR) {
                if (a.rank5) ptx::tma_load_5d_pair(dst, &tmap_x, afb_l, c0, wc, hc, dc, ht.n);
                else ptx::tma_load_4d_pair(dst, &tmap_x, afb_l, c0, wc, hc, ht.n);
              } else {
                if (a.rank5) ptx::tma_load_5d(dst, &tmap_x, afb, c0, wc, hc, dc, ht.n);
                else ptx::tma_load_4d(dst, &tmap_x, afb, c0, wc, hc, ht.n);
              }
              ++afills;
              if (++ast == a.a_slots) {
                ast = 0;
                aph ^= 1u;
              }
            }
      }
      if constexpr (PAIR) {
        pair_settle_ring(tail->afull, a.a_slots, &tail->peer_done_a, &tail->peer_fills_a, leader, afills,
                         a.timeout_ns, [&](long long) { return a.halo_bytes; });
      } else if (!ok) {
        for (int s = 0; s < a.a_slots; ++s) {
          const long long arms = afills / a.a_slots + (s < afills % a.a_slots ? 1 : 0);
          if (arms > 0) wait_drain(ptx::smem_u32(&tail->afull[s]), static_cast<uint32_t>((arms - 1) & 1), a.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (a pair's leader)
    if (leader && lane == 0) {
      int bst = 0, ast = 0;
      uint32_t bph = 0, aph = 0;
      bool ok = true;
      int t = 0;
      if (a.inject_stall)
        ok = wait_bounded(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected);
      // descriptors built once; moved by constant offsets below
      const uint64_t d_ring = ptx::smem_desc(ptx::smem_u32(bring), 16, a.sbo, a.layout_type);
      const uint64_t d_halo = ptx::smem_desc(ptx::smem_u32(halo), 16, a.sbo, a.layout_type);
      const uint64_t sub_off = desc_off(a.b_bytes), st_off = desc_off(a.stage_bytes);
      const uint64_t slot_off = desc_off(a.halo_slot_bytes);
      // a strip row (8 pixels x kc channels) is one swizzle atom: sbo bytes
      const uint64_t row_off = desc_off(static_cast<uint32_t>(a.dh) * a.sbo);
      const int ksteps = a.kc >> 4;
      for (int tile = unit; ok && tile < a.total_tiles; tile += nunits, ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag, a.timeout_ns,
                          kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * kHTAccStride;
        uint32_t accumulate = 0;
        uint64_t d_strip = 0;
        int kh = 0;  // height tap of the next K block (K blocks run kh-fastest)
        for (int q0 = 0; ok && q0 < Q; q0 += a.kbs) {
          const int nsub = min(a.kbs, Q - q0);
          if ((!a.w_resident || t == 0) &&
              !wait_bounded(ptx::smem_u32(&tail->full[bst]), bph, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          uint64_t dw = d_ring + static_cast<uint64_t>(bst) * st_off;
          for (int j = 0; j < nsub; ++j) {
            if (kh == 0) {
              if (!wait_bounded(ptx::smem_u32(&tail->afull[ast]), aph, abort_flag, a.timeout_ns, kSiteMmaFull)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
              d_strip = d_halo + static_cast<uint64_t>(ast) * slot_off;
            }
            // the view for kh starts kh*dh strip rows (swizzle atoms) down
            mma_sub<PAIR>(ksteps, d_tmem, dw, d_strip + static_cast<uint64_t>(kh) * row_off, a.idesc, accumulate);
            accumulate = 1;
            dw += sub_off;
            if (kh == a.kH - 1) {
              // last tap of this (cc, kd, kw): its strip slot is free once these MMAs complete
              if constexpr (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&tail->aempty[ast]), 3);
              else ptx::mma_commit(ptx::smem_u32(&tail->aempty[ast]));
              if (++ast == a.a_slots) {
                ast = 0;
                aph ^= 1u;
              }
              kh = 0;
            } else {
              ++kh;
            }
          }
          if (!ok) break;
          if (a.w_resident) continue;  // resident weights are never released
          if constexpr (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&tail->empty[bst]), 3);
          else ptx::mma_commit(ptx::smem_u32(&tail->empty[bst]));
          if (++bst == a.stages) {
            bst = 0;
            bph ^= 1u;
          }
        }
        if (ok) {
          if constexpr (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&tail->acc_full[acc]), 3);
          else ptx::mma_commit(ptx::smem_u32(&tail->acc_full[acc]));
        }
      }
      // every MMA this thread issued has completed once `drain` fires
      if constexpr (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&tail->drain), 1);
      else ptx::mma_commit(ptx::smem_u32(&tail->drain));
      wait_drain(ptx::smem_u32(&tail->drain), 0, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp works alone on its quarter of the channels: it converts a
    // 32-column chunk (its channels x 32 pixels) into its own slice of the
    // staging tile and stores that slice with one TMA store issued by its
    // lane 0, so no warp waits for another between chunks.
    const int q = warp & 3;          // tensor-memory lane quarter
    const int qch = mo / 4;          // channels per warp: 32 (M = 128) or 16 (M = 64)
    constexpr int kRowsPerChunk = kTEpiRows / kHTBlockW;  // 4 output rows per 32 columns
    int t = 0, chunk_seq = 0;
    for (int tile = unit; tile < a.total_tiles; tile += nunits, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      bool ok = wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                                  kSiteEpiAccFull);
      // the four warps leave together when one of them gave up
      ok = named_bar_and(1, 128, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const HaloTTile ht = decode_halo_t_tile(a, tile);
      const int o0 = ht.g * a.Og + ht.ot * o_tile + static_cast<int>(rank) * mo + q * qch;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc) * kHTAccStride;
      for (int c = 0; c < BP; c += kTEpiRows) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c), r);
        ptx::tmem_ld_wait();
        const int h = ht.h0 + (c / kTEpiRows) * kRowsPerChunk;
        if (h >= a.Ho) continue;  // the same for every epilogue thread
        uint8_t* buf = stage_y + (a.epi_bufs == 2 ? (chunk_seq & 1) : 0) * kTEpiBytes + q * kTEpiWarpBytes;
        // this warp's store that last read the slice (two chunks ago, or the
        // previous one with a single buffer) must be done with it
        if (lane == 0) {
          if (a.epi_bufs == 2) ptx::bulk_wait_group_read<1>();
          else ptx::bulk_wait_group_read<0>();
        }
        __syncwarp();
        // slice [4 rows][8 columns][qch channels]: M = 128: lane l holds
        // channel 32q + l; M = 64: lanes 0..15 hold channels 16q .. 16q+15
        // (the other 16 lanes are empty)
        if (lane < qch) {
          uint16_t* dst = reinterpret_cast<uint16_t*>(buf) + lane;
#pragma unroll
          for (int p = 0; p < kTEpiRows; ++p) dst[p * qch] = cvt1<BF16>(__uint_as_float(r[p]));
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (a.rank5) ptx::tma_store_5d(&tmap_y, ptx::smem_u32(buf), o0, ht.w0, h, ht.od, ht.n);
          else ptx::tma_store_4d(&tmap_y, ptx::smem_u32(buf), o0, ht.w0, h, ht.n);
          ptx::bulk_commit_group();
        }
        ++chunk_seq;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // a pair's accumulator buffer is reused once both CTAs' epilogues are done
        const uint32_t ae = ptx::smem_u32(&tail->acc_empty[acc]);
        if constexpr (PAIR) ptx::mbar_arrive_cluster(ptx::mapa_shared(ae, 0));
        else ptx::mbar_arrive(ae);
      }
    }
    // every store of this warp has finished (reading shared memory and writing y) before exit
    if (lane == 0) ptx::bulk_wait_group<0>();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) ptx::cluster_sync();  // the leader's MMAs (which read this CTA's smem) are complete
  ptx::tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) ptx::tmem_dealloc_pair(tmem_base, a.tmem_cols);
    else ptx::tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

}  // namespace convfwd
