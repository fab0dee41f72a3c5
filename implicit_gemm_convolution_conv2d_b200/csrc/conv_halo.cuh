// conv_halo.cuh -- tcgen05 implicit-GEMM convolution forward with input reuse
// in the plain orientation (rows = output pixels, columns = output channels):
// stride 1, C/G a multiple of 32, f16/bf16.
//
// A CTA owns a block of 16 x 8 output pixels (h x w) of one (n, od) output
// plane: GEMM rows m = r*8 + c for r < 16, c < 8 (a CTA pair stacks two such
// blocks, 32 x 8, and issues M = 256).  For each channel chunk (kc = 64 or 32
// channels), depth tap kd and width tap kw, ONE tiled TMA box brings the input
// column strip the block needs -- (16 + dh*(kH-1)) rows x 8 columns (shifted by
// kw*dw) x kc channels, zero-filled outside the image.  Every height tap kh
// then reads a view of it that starts kh*dh strip rows down: a strip row is 8
// pixels x kc*2 bytes, exactly one swizzle atom (1024 bytes with the 128-byte
// swizzle at kc = 64, 512 bytes with the 64-byte swizzle at kc = 32), so every
// view is a standard K-major operand on an atom boundary.  Each input pixel is
// fetched once per (chunk, kd, kw) instead of once per tap.
//
// The weights ([BN x kc] tiles, one per (chunk, tap)) stream through their
// own ring and the strips through theirs, from two producer threads, so that
// neither ring waits on the other.  Roles, bounded waits and the accumulator
// double-buffer are those of the other tensor-core kernels.  With PAIR, the
// leader issues tcgen05.mma.cta_group::2 and each CTA loads half of every
// weight tile and the strip of its own 16 rows.
#pragma once

#include "conv_tc.cuh"

namespace convfwd {

struct HaloTile {
  int g, n, od, h0, w0, nt;
};

__device__ __forceinline__ HaloTile decode_halo_tile(const TcArgs& a, int tile, int rank, bool pair) {
  HaloTile t;
  t.nt = tile % a.n_tiles;
  int q = tile / a.n_tiles;
  const int tw = q % a.tiles_w;
  q /= a.tiles_w;
  const int th = q % a.tiles_h;
  q /= a.tiles_h;
  const int plane = q % (a.N * a.Do);
  t.g = q / (a.N * a.Do);
  t.od = plane % a.Do;
  t.n = plane / a.Do;
  t.h0 = th * (pair ? 2 * a.tile_h : a.tile_h) + rank * a.tile_h;
  t.w0 = tw * a.tile_w;
  return t;
}

template <bool BF16, bool PAIR>
__global__ void __launch_bounds__(192, 1)
    conv_fwd_tc_halo_kernel(const __grid_constant__ CUtensorMap tmap_x,
                            const __grid_constant__ CUtensorMap tmap_w, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* halo = smem;                                        // a_slots x halo_slot_bytes
  uint8_t* bring = smem + a.a_slots * a.halo_slot_bytes;       // stages x (kbs x b_bytes)
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(bring + a.stages * a.stage_bytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
  const bool leader = rank == 0;

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
  const int unit = PAIR ? (blockIdx.x >> 1) : blockIdx.x;
  const int nunits = PAIR ? (gridDim.x >> 1) : gridDim.x;
  const int taps_hw = a.kH * a.kW;
  const uint32_t mult = PAIR ? 2u : 1u;

  // K blocks of a tile in issue order: q = ((cc * kD + kd) * kW + kw) * kH + kh.
  // A pipeline stage holds kbs consecutive K blocks (weight tiles); each
  // (cc, kd, kw) group has one strip in its own ring of a_slots slots.
  const int Q = a.cchunks * a.kD * taps_hw;
  if (warp == 0) {
    // ------------------------------------------------------------ producers
    // lane 0 streams the weight tiles, lane 1 the input strips, each on its
    // own ring; each arms a barrier only right before issuing every load it
    // covers, so a wait that gives up never leaves bytes expected that were
    // not requested.  (A pair's loads complete on the leader's barriers.)
    if (lane == 0) {
      int bst = 0;
      uint32_t bph = 0;
      long long bfills = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < a.total_tiles; tile += nunits) {
        const HaloTile ht = decode_halo_tile(a, tile, static_cast<int>(rank), PAIR);
        const int brow = ht.g * a.Og + ht.nt * a.BN + (PAIR ? static_cast<int>(rank) * (a.BN >> 1) : 0);
        int kh = 0, kw = 0, kd = 0, cc = 0;  // tap of the next K block
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
            if constexpr (PAIR) ptx::tma_load_2d_pair(sb, &tmap_w, fb_l, wtap(a, tap) * a.Cg + cc * a.kc, brow);
            else ptx::tma_load_2d(sb, &tmap_w, fb, wtap(a, tap) * a.Cg + cc * a.kc, brow);
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
        // settle every fill either issued
        const int fpt = (Q + a.kbs - 1) / a.kbs;
        pair_settle_ring(tail, a.stages, leader, bfills, a.timeout_ns, [&](long long k) {
          return static_cast<uint32_t>(min(a.kbs, Q - static_cast<int>(k % fpt) * a.kbs)) * a.b_bytes;
        });
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
        const HaloTile ht = decode_halo_tile(a, tile, static_cast<int>(rank), PAIR);
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
              const int wc = ht.w0 - a.pw + kw * a.dw, hc = ht.h0 - a.ph, dc = ht.od - a.pd + kd * a.dd;
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
      const uint64_t d_halo = ptx::smem_desc(ptx::smem_u32(halo), 16, a.sbo, a.layout_type);
      const uint64_t d_ring = ptx::smem_desc(ptx::smem_u32(bring), 16, a.sbo, a.layout_type);
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
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        uint32_t accumulate = 0;
        uint64_t d_strip = 0;
        int kh = 0;  // height tap of the next K block (K blocks run kh-fastest)
        for (int q0 = 0; ok && q0 < Q; q0 += a.kbs) {
          const int nsub = min(a.kbs, Q - q0);
          if (!wait_bounded(ptx::smem_u32(&tail->full[bst]), bph, abort_flag, a.timeout_ns, kSiteMmaFull)) {
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
            mma_sub<PAIR>(ksteps, d_tmem, d_strip + static_cast<uint64_t>(kh) * row_off, dw, a.idesc, accumulate);
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
      if constexpr (PAIR) ptx::mma_commit_pair(ptx::smem_u32(&tail->drain), 1);
      else ptx::mma_commit(ptx::smem_u32(&tail->drain));
      wait_drain(ptx::smem_u32(&tail->drain), 0, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int r = row >> 3, c = row & 7;
    uint16_t* __restrict__ y = static_cast<uint16_t*>(a.y);
    int t = 0;
    for (int tile = unit; tile < a.total_tiles; tile += nunits, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      if (!wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                             kSiteEpiAccFull))
        break;
      ptx::tc_fence_after();
      const HaloTile ht = decode_halo_tile(a, tile, static_cast<int>(rank), PAIR);
      const int h = ht.h0 + r, w = ht.w0 + c;
      const bool valid = h < a.Ho && w < a.Wo;
      const long long m = ((static_cast<long long>(ht.n) * a.Do + ht.od) * a.Ho + h) * a.Wo + w;
      const int n0 = ht.nt * a.BN;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
      const long long ybase = m * a.O + static_cast<long long>(ht.g) * a.Og;
      for (int cb = 0; cb < a.BN; cb += 32) {
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(taddr + cb, v);
        ptx::tmem_ld_wait();
        const int col0 = n0 + cb;
        const int nvalid = min(32, a.Og - col0);
        if (valid && nvalid > 0) {
          uint16_t* dst = y + ybase + col0;
          if (nvalid == 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 o;
              o.x = pack2<BF16>(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
              o.y = pack2<BF16>(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
              o.z = pack2<BF16>(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
              o.w = pack2<BF16>(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
              d4[j] = o;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nvalid) dst[j] = cvt1<BF16>(__uint_as_float(v[j]));
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        const uint32_t ae = ptx::smem_u32(&tail->acc_empty[acc]);
        if constexpr (PAIR) ptx::mbar_arrive_cluster(ptx::mapa_shared(ae, 0));
        else ptx::mbar_arrive(ae);
      }
    }
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) ptx::cluster_sync();
  ptx::tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) ptx::tmem_dealloc_pair(tmem_base, a.tmem_cols);
    else ptx::tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

}  // namespace convfwd
