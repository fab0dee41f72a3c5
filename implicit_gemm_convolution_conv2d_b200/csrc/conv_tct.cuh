// conv_tct.cuh -- tcgen05 implicit-GEMM convolution forward in the transposed
// (weight-stationary) orientation.
//
// The GEMM of the "Convolutions" tutorial (section 5, "Implicit GEMM") is
// y[m, o] = sum_k X[m, k] W[o, k] with m = (n, od, oh, ow), k = (kd, kh, kw, c).
// Its transpose y^T[o, m] = sum_k W[o, k] X[m, k] is the same sum with the
// operands swapped.  This kernel issues it that way round:
//   MMA M = 128 output channels      (A operand: a weight tile, K-major)
//   MMA N = BP output pixels (256)   (B operand: patch rows by TMA im2col, K-major)
// so that layers with 128 output channels per group still run the widest
// single-CTA instruction (128 x 256 x 16) instead of 128 x 128 x 16, which on
// B200 costs nearly as many cycles for half the work.  Both operands keep the
// layouts of the other TMA kernels (128-byte rows, K-major, swizzled); only
// their roles change.
//
// The accumulator holds y^T: tensor-memory lane = output channel, column =
// output pixel.  The epilogue therefore transposes through shared memory: a
// group of four warps reads 32 channels x 32 pixels each, writes them as 32
// pixel rows of a [32 pixels][128 channels] staging tile, and one thread
// stores the tile to y with a TMA tensor store (y viewed as [M][O]; rows
// beyond M are clipped by the tensor map).  Two staging tiles per group
// alternate so the next transpose overlaps the previous store, and two groups
// take alternate 32-pixel chunks (the epilogue, not the MMA, limits layers
// with a short reduction such as 3x1x1 over 64 channels).
//
// Warp roles (320 threads, one CTA per SM, static tile list):
//   warp 0      TMA producer (one thread): per K sub-block one weight tile
//               (128 x kc) and BP/128 im2col loads of 128 pixels x kc;
//   warp 1      TMEM allocator and MMA issuer (one thread);
//   warps 2..9  epilogue, groups 2..5 and 6..9; warp w reads tensor-memory
//               lanes 32*(w%4)..+31.
// Waits are bounded exactly as in the other tcgen05 kernels; each group's
// named barrier (1 or 2) is reached by exactly its four warps.
#pragma once

#include "conv_tc.cuh"

namespace convfwd {

constexpr int kTO = 128;                 // output channels per tile (MMA M)
constexpr int kTEpiRows = 32;            // pixels per staging tile
constexpr uint32_t kTEpiBytes = kTEpiRows * kTO * 2;  // 8 KB
constexpr int kTThreads = 192;
// The transposed im2col kernel runs two epilogue groups of four warps (even
// and odd 32-column chunks), each with its own staging tiles and store thread.
constexpr int kTEpiGroups = 2;
constexpr int kTTileThreads = 32 * (2 + 4 * kTEpiGroups);

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

template <bool BF16>
__global__ void __launch_bounds__(kTTileThreads, 1)
    conv_fwd_tc_t_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                         const __grid_constant__ CUtensorMap tmap_y, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_y = smem + static_cast<size_t>(a.stages) * a.stage_bytes;  // 2 per epilogue group
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(stage_y + 2 * kTEpiGroups * kTEpiBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BP = a.BN;                   // output pixels per tile (MMA N)
  const int halves = BP / kBM;           // im2col loads of 128 pixels per sub-block
  const uint32_t half_bytes = static_cast<uint32_t>(kBM * a.kc * 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->full[s]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->empty[s]), 1u);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&tail->acc_full[b]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->acc_empty[b]), 4u * kTEpiGroups);
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
  ptx::pdl_allow_next();  // setup done: the next launch may start its own
  ptx::pdl_wait_prev();   // the previous launch's writes are visible from here on
  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long fills = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x) {
        const TileCoord tc = decode_tile(a, tile);
        // corner of the im2col traversal of each 128-pixel half of the tile
        int hn[2], hw[2], hh[2], hd[2];
        for (int h = 0; h < halves; ++h) {
          int n, od, oh, ow;
          decode_pixel(a, static_cast<long long>(tc.mt) * BP + h * kBM, n, od, oh, ow);
          hn[h] = n;
          hw[h] = ow * a.sw - a.pw;
          hh[h] = oh * a.sh - a.ph;
          hd[h] = od * a.sd - a.pd;
        }
        const int orow = tc.g * a.Og + tc.nt * kTO;
        int tap = 0, cchunk = 0;
        for (int kb = 0; kb < a.kblocks; kb += a.kbs) {
          const int nsub = min(a.kbs, a.kblocks - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = ptx::smem_u32(&tail->full[stage]);
          ptx::mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nsub) * (a.a_bytes + a.b_bytes));
          for (int j = 0; j < nsub; ++j) {
            const uint32_t sa = ptx::smem_u32(smem + stage * a.stage_bytes + j * a.sub_bytes);
            const uint32_t sb = sa + a.a_bytes;
            const int kw = tap % a.kW;
            const int kh = (tap / a.kW) % a.kH;
            const int kd = tap / (a.kW * a.kH);
            const int c0 = tc.g * a.Cg + cchunk * a.kc;
            ptx::tma_load_2d(sa, &tmap_w, fb, wtap(a, tap) * a.Cg + cchunk * a.kc, orow);
            for (int h = 0; h < halves; ++h) {
              const uint32_t dst = sb + static_cast<uint32_t>(h) * half_bytes;
              if (a.rank5)
                ptx::tma_load_im2col_5d(dst, &tmap_x, fb, c0, hw[h], hh[h], hd[h], hn[h],
                                        static_cast<uint16_t>(kw * a.dw), static_cast<uint16_t>(kh * a.dh),
                                        static_cast<uint16_t>(kd * a.dd));
              else
                ptx::tma_load_im2col_4d(dst, &tmap_x, fb, c0, hw[h], hh[h], hn[h],
                                        static_cast<uint16_t>(kw * a.dw), static_cast<uint16_t>(kh * a.dh));
            }
            if (++cchunk == a.cchunks) {
              cchunk = 0;
              ++tap;
            }
          }
          ++fills;
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
            wait_drain(ptx::smem_u32(&tail->full[s]), static_cast<uint32_t>((arms - 1) & 1), a.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int t = 0;
      if (a.inject_stall)
        ok = wait_bounded(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected);
      // descriptors built once; moved by constant offsets below
      const uint64_t d_ring = ptx::smem_desc(ptx::smem_u32(smem), 16, a.sbo, a.layout_type);
      const uint64_t a_off = desc_off(a.a_bytes), sub_off = desc_off(a.sub_bytes), st_off = desc_off(a.stage_bytes);
      const int ksteps = a.kc >> 4;
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
        for (int kb = 0; kb < a.kblocks; kb += a.kbs) {
          const int nsub = min(a.kbs, a.kblocks - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          uint64_t da = d_ring + static_cast<uint64_t>(stage) * st_off;
          for (int j = 0; j < nsub; ++j) {
            mma_sub<false>(ksteps, d_tmem, da, da + a_off, a.idesc, (kb + j) != 0 ? 1u : 0u);
            da += sub_off;
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
    // group g = (warp - 2) / 4 takes 32-column chunks g, g + 2, ...; its four
    // warps cover the four tensor-memory lane quarters and synchronise on
    // named barrier 1 + g
    const int q = warp & 3;                  // tensor-memory lane quarter: channels 32q .. 32q+31
    const int grp = (warp - 2) >> 2;
    const uint32_t bar_id = 1u + static_cast<uint32_t>(grp);
    const bool store_thread = warp == 2 + 4 * grp && lane == 0;
    uint8_t* const stage_g = stage_y + 2 * grp * kTEpiBytes;
    int t = 0, chunk_seq = 0;
    for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      bool ok = wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                                  kSiteEpiAccFull);
      // the group's four warps agree before any of them enters the named
      // barriers below: a warp whose wait gave up must not leave the others waiting
      ok = named_bar_and(bar_id, 128, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const TileCoord tc = decode_tile(a, tile);
      const long long m0 = static_cast<long long>(tc.mt) * BP;
      const int o0 = tc.g * a.Og + tc.nt * kTO;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BP);
      for (int c = grp * kTEpiRows; c < BP; c += kTEpiGroups * kTEpiRows) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c), r);
        ptx::tmem_ld_wait();
        const long long mrow = m0 + c;
        if (mrow >= a.M) continue;           // the same for every thread of the group
        uint8_t* buf = stage_g + (chunk_seq & 1) * kTEpiBytes;
        // the store issued two chunks ago read this buffer; it must be done
        if (store_thread) ptx::bulk_wait_group_read<1>();
        named_bar_sync(bar_id, 128);
        uint16_t* dst = reinterpret_cast<uint16_t*>(buf) + q * 32 + lane;
#pragma unroll
        for (int p = 0; p < kTEpiRows; ++p) dst[p * kTO] = cvt1<BF16>(__uint_as_float(r[p]));
        ptx::fence_proxy_async_smem();
        named_bar_sync(bar_id, 128);
        if (store_thread) {
          ptx::tma_store_2d(&tmap_y, ptx::smem_u32(buf), o0, static_cast<int32_t>(mrow));
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
