// conv_halo_t.cuh -- tcgen05 implicit-GEMM convolution forward, transposed
// orientation with input-halo reuse (stride 1, C/G % 64 == 0, O/G % 128 == 0).
//
// The product is issued as y^T[o, m] = sum_k W[o, k] X[m, k] (see
// conv_tct.cuh): MMA M = 128 output channels (A = a weight tile), N = 256
// output pixels (B = patch rows).  The 256 pixels are a block of 32 x 8
// output pixels (h x w) of one (n, od) plane, and B is not loaded per tap:
// for each 64-channel chunk, depth tap kd and width tap kw, ONE tiled TMA box
// brings the input column strip the block needs -- (32 + dh*(kH-1)) rows x 8
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
// Epilogue: the accumulator holds [128 channels][256 pixels]; 32 columns are
// 4 output rows x 8 output columns.  Four warps transpose each such chunk into
// a [4][8][128] staging tile and one thread stores it with a 4-D / 5-D TMA
// tensor store on y viewed as [N, (Do,) Ho, Wo, O], which clips the rows and
// columns of the block that fall outside the output.
#pragma once

#include "conv_halo.cuh"
#include "conv_tct.cuh"

namespace convfwd {

constexpr int kHTBlockH = 32, kHTBlockW = 8;  // output block: MMA N = 256 pixels

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

template <bool BF16>
__global__ void __launch_bounds__(kTThreads, 1)
    conv_fwd_tc_halo_t_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                              const __grid_constant__ CUtensorMap tmap_y, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* halo = smem;                                              // a_slots x halo_slot_bytes
  uint8_t* bring = smem + a.a_slots * a.halo_slot_bytes;             // stages x (kbs weight tiles)
  uint8_t* stage_y = bring + static_cast<size_t>(a.stages) * a.stage_bytes;  // 2 staging tiles
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(stage_y + 2 * kTEpiBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

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
      ptx::mbar_init(ptx::smem_u32(&tail->acc_empty[b]), 4u);
    }
    ptx::mbar_init(ptx::smem_u32(&tail->drain), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->stall), 1u);
    tail->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_y);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&tail->tmem_base), a.tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;
  const int taps_hw = a.kH * a.kW;
  const int BP = a.BN;  // 256 output pixels per tile

  // K blocks of a tile in issue order: q = ((cc * kD + kd) * kW + kw) * kH + kh.
  // A pipeline stage holds up to kbs consecutive K blocks (weight tiles); each
  // (cc, kd, kw) group has one strip, loaded before its first K block.  With
  // kbs <= kH a stage spans at most two groups, so two strip slots suffice.
  const int Q = a.cchunks * a.kD * taps_hw;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int bst = 0, ast = 0;
      uint32_t bph = 0, aph = 0;
      long long bfills = 0, afills = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x) {
        const HaloTTile ht = decode_halo_t_tile(a, tile);
        const int orow = ht.g * a.Og + ht.ot * kTO;
        for (int q0 = 0; ok && q0 < Q; q0 += a.kbs) {
          const int nsub = min(a.kbs, Q - q0);
          if (!wait_bounded(ptx::smem_u32(&tail->empty[bst]), bph ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          // halo boxes first: a wait that gives up here leaves no stage armed
          for (int j = 0; j < nsub; ++j) {
            const int q = q0 + j;
            if (q % a.kH != 0) continue;
            const int grp = q / a.kH;
            const int kw = grp % a.kW, kd = (grp / a.kW) % a.kD, cc = grp / (a.kW * a.kD);
            if (!wait_bounded(ptx::smem_u32(&tail->aempty[ast]), aph ^ 1u, abort_flag, a.timeout_ns,
                              kSiteProducerEmpty)) {
              ok = false;
              break;
            }
            const uint32_t afb = ptx::smem_u32(&tail->afull[ast]);
            ptx::mbar_arrive_expect_tx(afb, a.halo_bytes);
            const uint32_t dst = ptx::smem_u32(halo + ast * a.halo_slot_bytes);
            const int c0 = ht.g * a.Cg + cc * 64;
            const int wc = ht.w0 - a.pw + kw * a.dw, hc = ht.h0 - a.ph, dc = ht.od - a.pd + kd * a.dd;
            if (a.rank5) ptx::tma_load_5d(dst, &tmap_x, afb, c0, wc, hc, dc, ht.n);
            else ptx::tma_load_4d(dst, &tmap_x, afb, c0, wc, hc, ht.n);
            ++afills;
            if (++ast == a.a_slots) {
              ast = 0;
              aph ^= 1u;
            }
          }
          if (!ok) break;
          // then the stage's weight tiles, armed for exactly what is issued
          const uint32_t fb = ptx::smem_u32(&tail->full[bst]);
          ptx::mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nsub) * a.b_bytes);
          for (int j = 0; j < nsub; ++j) {
            const int q = q0 + j;
            const int kh = q % a.kH, grp = q / a.kH;
            const int kw = grp % a.kW, kd = (grp / a.kW) % a.kD, cc = grp / (a.kW * a.kD);
            const uint32_t sb = ptx::smem_u32(bring + bst * a.stage_bytes + j * a.b_bytes);
            const int tap = (kd * a.kH + kh) * a.kW + kw;  // weight layout (kd, kh, kw)
            ptx::tma_load_2d(sb, &tmap_w, fb, tap * a.Cg + cc * 64, orow);
          }
          ++bfills;
          if (++bst == a.stages) {
            bst = 0;
            bph ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < a.stages; ++s) {
          const long long arms = bfills / a.stages + (s < bfills % a.stages ? 1 : 0);
          if (arms > 0) wait_drain(ptx::smem_u32(&tail->full[s]), static_cast<uint32_t>((arms - 1) & 1), a.timeout_ns);
        }
        for (int s = 0; s < a.a_slots; ++s) {
          const long long arms = afills / a.a_slots + (s < afills % a.a_slots ? 1 : 0);
          if (arms > 0) wait_drain(ptx::smem_u32(&tail->afull[s]), static_cast<uint32_t>((arms - 1) & 1), a.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int bst = 0, ast = 0;
      uint32_t bph = 0, aph = 0;
      bool ok = true;
      int t = 0;
      if (a.inject_stall)
        ok = wait_bounded(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected);
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x, ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag, a.timeout_ns,
                          kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BP);
        uint32_t accumulate = 0;
        uint32_t hbase = 0;
        for (int q0 = 0; ok && q0 < Q; q0 += a.kbs) {
          const int nsub = min(a.kbs, Q - q0);
          if (!wait_bounded(ptx::smem_u32(&tail->full[bst]), bph, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          for (int j = 0; j < nsub; ++j) {
            const int q = q0 + j;
            const int kh = q % a.kH;
            if (kh == 0) {
              if (!wait_bounded(ptx::smem_u32(&tail->afull[ast]), aph, abort_flag, a.timeout_ns, kSiteMmaFull)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
              hbase = ptx::smem_u32(halo + ast * a.halo_slot_bytes);
            }
            // strip rows are 8 pixels = 1024 bytes: the view for kh starts kh*dh atoms down
            const uint32_t view = hbase + static_cast<uint32_t>(kh * a.dh) * 1024u;
            const uint32_t sw = ptx::smem_u32(bring + bst * a.stage_bytes + j * a.b_bytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t da = ptx::smem_desc(sw + k * 32, 16, 1024, 2);
              const uint64_t db = ptx::smem_desc(view + k * 32, 16, 1024, 2);
              ptx::mma_f16(d_tmem, da, db, a.idesc, accumulate);
              accumulate = 1;
            }
            if (kh == a.kH - 1) {
              // last tap of this (cc, kd, kw): its strip slot is free once these MMAs complete
              ptx::mma_commit(ptx::smem_u32(&tail->aempty[ast]));
              if (++ast == a.a_slots) {
                ast = 0;
                aph ^= 1u;
              }
            }
          }
          if (!ok) break;
          ptx::mma_commit(ptx::smem_u32(&tail->empty[bst]));
          if (++bst == a.stages) {
            bst = 0;
            bph ^= 1u;
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
    const int q = warp & 3;  // tensor-memory lane quarter: channels 32q .. 32q+31
    const bool store_thread = warp == 2 && lane == 0;
    constexpr int kRowsPerChunk = kTEpiRows / kHTBlockW;  // 4 output rows per 32 columns
    int t = 0, chunk_seq = 0;
    for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      bool ok = wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                                  kSiteEpiAccFull);
      // the four warps agree before any of them enters the named barriers
      // below: a warp whose wait gave up must not leave the others waiting
      ok = named_bar_and(1, 128, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const HaloTTile ht = decode_halo_t_tile(a, tile);
      const int o0 = ht.g * a.Og + ht.ot * kTO;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BP);
      for (int c = 0; c < BP; c += kTEpiRows) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c), r);
        ptx::tmem_ld_wait();
        const int h = ht.h0 + (c / kTEpiRows) * kRowsPerChunk;
        if (h >= a.Ho) continue;  // the same for every epilogue thread
        uint8_t* buf = stage_y + (chunk_seq & 1) * kTEpiBytes;
        // the store issued two chunks ago read this buffer; it must be done
        if (store_thread) ptx::bulk_wait_group_read<1>();
        named_bar_sync(1, 128);
        uint16_t* dst = reinterpret_cast<uint16_t*>(buf) + q * 32 + lane;
#pragma unroll
        for (int p = 0; p < kTEpiRows; ++p) dst[p * kTO] = cvt1<BF16>(__uint_as_float(r[p]));
        ptx::fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (store_thread) {
          if (a.rank5) ptx::tma_store_5d(&tmap_y, ptx::smem_u32(buf), o0, ht.w0, h, ht.od, ht.n);
          else ptx::tma_store_4d(&tmap_y, ptx::smem_u32(buf), o0, ht.w0, h, ht.n);
          ptx::bulk_commit_group();
        }
        ++chunk_seq;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&tail->acc_empty[acc]));
    }
    // every store has finished (reading shared memory and writing y) before exit
    if (store_thread) ptx::bulk_wait_group<0>();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem_base, a.tmem_cols);
}

}  // namespace convfwd
