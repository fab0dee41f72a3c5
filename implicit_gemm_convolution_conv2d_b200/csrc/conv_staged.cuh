// conv_staged.cuh -- tcgen05 implicit-GEMM convolution forward for channel
// counts that neither TMA nor the MMA's swizzled layouts can address (a pixel
// pitch of C*2 bytes that is not a multiple of 16), f16/bf16, stride 1,
// O <= 128, one group.
//
// The product is issued transposed, y^T[o, m] = sum_k W[o, k] X[m, k]: MMA
// M = 128 output-channel rows, N = 8 * tile_h output pixels, a block of
// tile_h x 8 pixels (h x w) of one (n, od) output plane, as in the transposed
// halo kernel.
//
// Operands live in shared memory in the canonical K-major layout WITHOUT
// swizzle: a core matrix is 8 rows x 16 bytes (8 channels), its rows 16 bytes
// apart; the descriptor's SBO steps between 8-row groups, its LBO between the
// two 8-channel halves of a 16-wide K step.  Builder warps realign, for each
// (depth tap kd, 16-channel chunk), the input region the block needs --
// Hr = tile_h + dh*(kH-1) rows x Wr = 8 + dw*(kW-1) columns, each pixel's 16
// channels as two 16-byte halves in two planes -- and the weights of the kH*kW
// taps of that kd and chunk.  Every (kh, kw) tap then reads the region through
// a view: N-group j (output row j of the block) starts at region pixel
// (j + kh*dh, kw*dw), i.e. start = plane + (kh*dh*Wr + kw*dw)*16 and SBO =
// Wr*16, so one staged region serves all kH*kW taps.  The largest pixel a view
// reaches is (Hr-1)*Wr + Wr-1, the region's last.
//
// Realignment: 8 channels starting at element e come from the one or two
// aligned 16-byte blocks holding them (see st_fetch); a builder thread issues
// the loads of its whole batch of units before it extracts and stores any.
// Channels >= C and pixels outside the input are zeros.  A tap's weights
// take ceil(O/8) 8-row groups of a slot and the next tap follows at once:
// the MMA's rows >= O read whatever lies beyond (the next tap, or slack at the
// end of the weight area) and land in accumulator lanes the epilogue never
// stores.
//
// Roles: 20 builder warps (every builder thread waits on the slot's `empty`
// barrier, fills its share, fences the async proxy and arrives on `full`),
// one MMA-issuing thread (warp 20), four epilogue warps (21..24, tensor-memory
// lane quarter warp & 3) that convert 32-column chunks and store y with
// 16-bit stores (y's rows are O*2 bytes apart, not a TMA stride).  Two
// accumulators of 256 columns; every wait is bounded.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "conv_tc.cuh"
#include "conv_tct.cuh"  // named_bar_and
#include "ptx.cuh"

namespace convfwd {

// The builders are latency-bound: 8, 12, 16 and 20 warps took 0.205, 0.176,
// 0.152 and 0.148 ms on (4,32^3,65)->65.
constexpr int kStBuilderWarps = 20;
constexpr int kStBuilders = 32 * kStBuilderWarps;
constexpr int kStMmaWarp = kStBuilderWarps;         // warp 20
constexpr int kStThreads = 32 * (kStBuilderWarps + 1 + 4);
constexpr uint32_t kStAGroupBytes = 256;           // 8 weight rows x 16 channels (two 128-byte halves)
constexpr uint32_t kStAccStride = 256;              // tensor-memory columns per accumulator
constexpr int kStBlockW = 8;

struct StArgs {
  int N, D, H, W, C, O;
  int kD, kH, kW;
  int pd, ph, pw;        // padding below each dimension (stride 1)
  int dd, dh, dw;        // dilation
  int Do, Ho, Wo;
  long long K;           // kD*kH*kW*C: one output channel's weights
  long long x_blocks, w_blocks;  // 16-byte blocks holding x's / w's elements
  int raw;               // 1: inputs and weights staged raw in shared memory once per (block, kd)
  uint32_t rx_row;       // raw mode: bytes per staged input row (its 16-byte cover, rounded up)
  uint32_t rw_row;       // raw mode: bytes per staged weight row
  uint32_t raw_x_off;    // raw mode: byte offsets of the staged input rows and weight rows
  uint32_t raw_w_off;
  uint32_t tail_off;     // byte offset of the barriers
  int tile_h;            // output rows of a block (N = 8 * tile_h)
  int tiles_h, tiles_w, total_tiles;
  int nc16;              // 16-channel chunks: ceil(C / 16)
  int pix_stride;        // raw mode: region unit q packs pixel (q * pix_stride) mod (Hr*Wr), a stride
                         // coprime to Hr*Wr chosen on the host to spread the builders' shared-memory
                         // reads over the banks
  int Hr, Wr;            // staged region rows / columns
  uint32_t plane_bytes;  // Hr * Wr * 16
  uint32_t tap_bytes;    // one tap's weights in a slot: ceil(O/8) 8-row groups
  uint32_t a_bytes;      // kH * kW * tap_bytes + the (16 - ceil(O/8)) groups the last tap's MMA reads past them
  uint32_t stage_bytes;  // a_bytes + 2 * plane_bytes, rounded up to 128
  int stages;
  uint32_t idesc;
  uint32_t tmem_cols;
  unsigned long long timeout_ns;
  int inject_stall;
  const void* x;
  const void* w;
  void* y;
};

struct __align__(8) StTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint64_t stall;  // never arrived on (the injected-timeout test waits here)
  uint32_t tmem_base;
  volatile int abort_flag;
};

struct StTile {
  int n, od, h0, w0;
};

// Tile -> (image, output depth, block origin); blocks along w vary fastest so
// that CTAs working at the same time share input rows through L2.
__device__ __forceinline__ StTile st_decode(const StArgs& a, int tile) {
  StTile t;
  const int tw = tile % a.tiles_w;
  int q = tile / a.tiles_w;
  const int th = q % a.tiles_h;
  q /= a.tiles_h;
  t.od = q % a.Do;
  t.n = q / a.Do;
  t.h0 = th * a.tile_h;
  t.w0 = tw * kStBlockW;
  return t;
}

// One 16-byte unit of a pipeline slot: 8 consecutive 16-bit elements starting
// at element e of x or w, of which the first `nval` exist (the rest are
// channels >= C and read as zeros).  The unit is fetched as the aligned
// 16-byte block holding element e and, when the eight elements run past it,
// the next block; the elements are picked out afterwards.  A block is read
// only if the tensor's data reaches into it (every block before the last one
// holding data); a unit that would need a block past that (the last few
// elements of the tensor) takes element loads instead.  Fetching every unit
// of a batch before extracting any keeps all their loads in flight at once.
struct StUnit {
  uint4 lo, hi;
  uint32_t dst;   // shared-memory address of the unit, or kStNoUnit
  uint32_t meta;  // byte offset of element e in its block (bits 0-3), nval (bits 4-7); kStZero: zeros
};
constexpr uint32_t kStNoUnit = 0xffffffffu;
constexpr uint32_t kStZero = 0x100u;

__device__ __forceinline__ void st_fetch(StUnit& u, const uint16_t* __restrict__ p, long long e, int nval,
                                         long long nblocks) {
  if (nval <= 0) {
    u.meta = kStZero;
    return;
  }
  nval = min(nval, 8);
  const long long b = e >> 3;
  const uint32_t off = static_cast<uint32_t>(e & 7) * 2u;
  const bool two = off + 2u * static_cast<uint32_t>(nval) > 16u;
  if (b + (two ? 2 : 1) <= nblocks) {
    const uint4* bp = reinterpret_cast<const uint4*>(p) + b;
    u.lo = __ldg(bp);
    u.hi = two ? __ldg(bp + 1) : make_uint4(0u, 0u, 0u, 0u);
    u.meta = off | (static_cast<uint32_t>(nval) << 4);
  } else {
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = i < nval ? static_cast<uint32_t>(__ldg(p + e + i)) : 0u;
    u.lo = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
    u.meta = 8u << 4;  // offset 0, all eight taken as loaded
  }
}

// The 16 bytes at the unit's offset within lo:hi (word selects and a 16-bit
// funnel shift), elements >= nval cleared.
__device__ __forceinline__ uint4 st_extract(const StUnit& u) {
  if (u.meta & kStZero) return make_uint4(0u, 0u, 0u, 0u);
  const uint32_t off = u.meta & 15u, nval = (u.meta >> 4) & 15u;
  uint4 v;
  if (off == 0) {
    v = u.lo;
  } else {
    const bool w2 = (off & 8u) != 0, w1 = (off & 4u) != 0;
    // words off/4 .. off/4 + 4 of the 32 bytes
    const uint32_t t0 = w2 ? u.lo.z : u.lo.x, t1 = w2 ? u.lo.w : u.lo.y, t2 = w2 ? u.hi.x : u.lo.z,
                   t3 = w2 ? u.hi.y : u.lo.w, t4 = w2 ? u.hi.z : u.hi.x, t5 = w2 ? u.hi.w : u.hi.y;
    const uint32_t v0 = w1 ? t1 : t0, v1 = w1 ? t2 : t1, v2 = w1 ? t3 : t2, v3 = w1 ? t4 : t3, v4 = w1 ? t5 : t4;
    const uint32_t sh = (off & 2u) * 8u;
    v = make_uint4(__funnelshift_r(v0, v1, sh), __funnelshift_r(v1, v2, sh), __funnelshift_r(v2, v3, sh),
                   __funnelshift_r(v3, v4, sh));
  }
  return nval >= 8 ? v : mask8(v, (1u << nval) - 1u);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

constexpr int kStBatch = 3;  // units a builder thread has in flight

// Builder thread `bt`'s share of one pipeline slot: the region of depth tap kd
// and channel chunk cc for block t (units 0 .. 2*Hr*Wr-1: pixel u/2, channel
// half u&1) and the weights of that kd and chunk (the rest: tap, half, then
// output channel fastest, so that a warp's 16-byte stores fill whole 128-byte
// rows of the weight tiles).
__device__ __forceinline__ void st_build(const StArgs& a, const StTile& t, int kd, int cc, uint32_t sa, int bt) {
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  const uint16_t* __restrict__ w = static_cast<const uint16_t*>(a.w);
  const uint32_t sb = sa + a.a_bytes;  // region planes (sa: weights, taps x [16 groups][2 halves][8 rows][16 B])
  const int taps_hw = a.kH * a.kW;
  const int nB = 2 * a.Hr * a.Wr;
  const int total = nB + taps_hw * a.O * 2;
  const int id = t.od - a.pd + kd * a.dd;
  const bool plane_ok = static_cast<unsigned>(id) < static_cast<unsigned>(a.D);
  const long long xrow0 = (static_cast<long long>(t.n) * a.D + (plane_ok ? id : 0)) * a.H;  // input row of ih = 0
  const long long wkd = static_cast<long long>(kd) * taps_hw * a.C;  // tap (kd, 0, 0) within a weight row
  for (int base = bt; base < total; base += kStBatch * kStBuilders) {
    StUnit un[kStBatch];
#pragma unroll
    for (int i = 0; i < kStBatch; ++i) {
      const int u = base + i * kStBuilders;
      un[i].dst = kStNoUnit;
      un[i].meta = kStZero;
      if (u < nB) {
        const int kk = u & 1, pix = u >> 1;
        const int r = pix / a.Wr, c = pix - r * a.Wr;
        const int ih = t.h0 - a.ph + r, iw = t.w0 - a.pw + c;
        const int c0 = cc * 16 + kk * 8;
        un[i].dst = sb + static_cast<uint32_t>(kk) * a.plane_bytes + static_cast<uint32_t>(pix) * 16u;
        if (plane_ok && static_cast<unsigned>(ih) < static_cast<unsigned>(a.H) &&
            static_cast<unsigned>(iw) < static_cast<unsigned>(a.W))
          st_fetch(un[i], x, ((xrow0 + ih) * a.W + iw) * a.C + c0, a.C - c0, a.x_blocks);
      } else if (u < total) {
        const int q = u - nB;
        const int o = q % a.O, rest = q / a.O;
        const int kk = rest & 1, tap = rest >> 1;
        const int c0 = cc * 16 + kk * 8;
        un[i].dst = sa + static_cast<uint32_t>(tap) * a.tap_bytes + static_cast<uint32_t>(o >> 3) * 256u +
                    static_cast<uint32_t>(kk) * 128u + static_cast<uint32_t>(o & 7) * 16u;
        st_fetch(un[i], w, static_cast<long long>(o) * a.K + wkd + static_cast<long long>(tap) * a.C + c0, a.C - c0,
                 a.w_blocks);
      }
    }
#pragma unroll
    for (int i = 0; i < kStBatch; ++i)
      if (un[i].dst != kStNoUnit) st_shared_v4(un[i].dst, st_extract(un[i]));
  }
}

__device__ __forceinline__ uint4 st_lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// 16 bytes global -> shared, asynchronous (both addresses 16-byte aligned).
__device__ __forceinline__ void st_cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Raw mode, step 1 (every builder thread, once per (block, kd)): the input
// rows of the region -- their in-range pixels, as the aligned 16-byte blocks
// covering them -- and every output channel's weights of this kd (kH*kW*C
// elements, the same cover) copied to shared memory with coalesced 16-byte
// asynchronous copies: warp w takes rows w, w + 8, ..., its lanes consecutive
// blocks.  The caller waits for the copies and synchronises the builders.
__device__ __forceinline__ void st_stage_raw(const StArgs& a, const StTile& t, int kd, uint32_t raw_x, uint32_t raw_w,
                                             int bt) {
  const uint4* __restrict__ xb = static_cast<const uint4*>(a.x);
  const uint4* __restrict__ wb = static_cast<const uint4*>(a.w);
  const int warp = bt >> 5, lane = bt & 31;
  const int id = t.od - a.pd + kd * a.dd;
  const bool plane_ok = static_cast<unsigned>(id) < static_cast<unsigned>(a.D);
  const long long xrow0 = (static_cast<long long>(t.n) * a.D + (plane_ok ? id : 0)) * a.H;
  const int iw_lo = max(0, t.w0 - a.pw), iw_hi = min(a.W, t.w0 - a.pw + a.Wr);
  const long long seg = static_cast<long long>(a.kH) * a.kW * a.C;  // one output channel's weights of a kd
  for (int row = warp; row < a.Hr + a.O; row += kStBuilderWarps) {
    long long e_lo, e_hi;
    uint32_t dst;
    const uint4* src;
    if (row < a.Hr) {
      const int ih = t.h0 - a.ph + row;
      if (!plane_ok || ih < 0 || ih >= a.H || iw_lo >= iw_hi) continue;  // the same for the whole warp
      const long long rowe = (xrow0 + ih) * a.W * static_cast<long long>(a.C);
      e_lo = rowe + static_cast<long long>(iw_lo) * a.C;
      e_hi = rowe + static_cast<long long>(iw_hi) * a.C;
      dst = raw_x + static_cast<uint32_t>(row) * a.rx_row;
      src = xb;
    } else {
      const int o = row - a.Hr;
      e_lo = static_cast<long long>(o) * a.K + kd * seg;
      e_hi = e_lo + seg;
      dst = raw_w + static_cast<uint32_t>(o) * a.rw_row;
      src = wb;
    }
    const long long b_lo = (2 * e_lo) >> 4, b_hi = (2 * e_hi + 15) >> 4;
    const int nb = static_cast<int>(b_hi - b_lo);
    for (int j = lane; j < nb; j += 32) st_cp_async16(dst + static_cast<uint32_t>(j) * 16u, src + b_lo + j);
  }
}

// Raw mode, step 2: each builder thread's units of the (block, kd) slots,
// decoded once for the nc16 slots of the pair (a slot's units differ only by
// the 16-channel chunk: 32 bytes further along every staged row).  Unit i of
// thread bt is u = bt + i * kStBuilders (the numbering of st_build); at most
// kStBatch units a thread (the planner checks it).  base: the staged address
// of channel 8*kk of the unit's pixel / weight row for chunk 0; dst: its place
// in a slot; valid bit i: the unit reads staged data (else it stores zeros);
// kk bit i: the unit's channel half.
struct StPre {
  uint32_t base[kStBatch];
  uint32_t dst[kStBatch];
  uint32_t valid, kk, used;
};

__device__ __forceinline__ void st_pre_raw(const StArgs& a, const StTile& t, int kd, uint32_t raw_x, uint32_t raw_w,
                                           int bt, StPre& pr) {
  const int taps_hw = a.kH * a.kW;
  const int nB = 2 * a.Hr * a.Wr;
  const int total = nB + taps_hw * a.O * 2;
  const int id = t.od - a.pd + kd * a.dd;
  const bool plane_ok = static_cast<unsigned>(id) < static_cast<unsigned>(a.D);
  const int iw_lo = max(0, t.w0 - a.pw);
  const long long xrow0 = (static_cast<long long>(t.n) * a.D + (plane_ok ? id : 0)) * a.H;
  const uint32_t wc8 = static_cast<uint32_t>((static_cast<long long>(a.W) * a.C) & 7);
  const uint32_t k8 = static_cast<uint32_t>(a.K & 7);
  const uint32_t seg8 = static_cast<uint32_t>((static_cast<long long>(taps_hw) * a.C) & 7);
  pr.valid = pr.kk = pr.used = 0u;
#pragma unroll
  for (int i = 0; i < kStBatch; ++i) {
    const int u = bt + i * kStBuilders;
    pr.base[i] = 0u;
    pr.dst[i] = 0u;
    if (u < nB) {
      const int kk = u & 1, pix = static_cast<int>((static_cast<long long>(u >> 1) * a.pix_stride) % (a.Hr * a.Wr));
      const int r = pix / a.Wr, c = pix - r * a.Wr;
      const int ih = t.h0 - a.ph + r, iw = t.w0 - a.pw + c;
      pr.used |= 1u << i;
      pr.kk |= static_cast<uint32_t>(kk) << i;
      pr.dst[i] = a.a_bytes + static_cast<uint32_t>(kk) * a.plane_bytes + static_cast<uint32_t>(pix) * 16u;
      if (plane_ok && static_cast<unsigned>(ih) < static_cast<unsigned>(a.H) &&
          static_cast<unsigned>(iw) < static_cast<unsigned>(a.W)) {
        // (2 * (row element offset + iw_lo*C)) mod 16, in 32-bit arithmetic mod 8
        const uint32_t s0 = (2u * ((static_cast<uint32_t>(xrow0 + ih) & 7u) * wc8 + static_cast<uint32_t>(iw_lo * a.C))) & 15u;
        pr.base[i] = raw_x + static_cast<uint32_t>(r) * a.rx_row + s0 + 2u * static_cast<uint32_t>((iw - iw_lo) * a.C) +
                     16u * static_cast<uint32_t>(kk);
        pr.valid |= 1u << i;
      }
    } else if (u < total) {
      const int q = u - nB;
      const int o = q % a.O, rest = q / a.O;
      const int kk = rest & 1, tap = rest >> 1;
      pr.used |= 1u << i;
      pr.kk |= static_cast<uint32_t>(kk) << i;
      pr.dst[i] = static_cast<uint32_t>(tap) * a.tap_bytes + static_cast<uint32_t>(o >> 3) * 256u +
                  static_cast<uint32_t>(kk) * 128u + static_cast<uint32_t>(o & 7) * 16u;
      const uint32_t s0 = (2u * ((static_cast<uint32_t>(o) & 7u) * k8 + static_cast<uint32_t>(kd) * seg8)) & 15u;
      pr.base[i] = raw_w + static_cast<uint32_t>(o) * a.rw_row + s0 + 2u * static_cast<uint32_t>(tap * a.C) +
                   16u * static_cast<uint32_t>(kk);
      pr.valid |= 1u << i;
    }
  }
}

// Raw mode, step 3: the slot of chunk cc, from the decoded units.
__device__ __forceinline__ void st_pack_pre(const StArgs& a, const StPre& pr, int cc, uint32_t slot) {
  StUnit un[kStBatch];
#pragma unroll
  for (int i = 0; i < kStBatch; ++i) {
    un[i].meta = kStZero;
    const int nval = a.C - (cc * 16 + static_cast<int>((pr.kk >> i) & 1u) * 8);
    if (((pr.valid >> i) & 1u) && nval > 0) {
      const int nv = min(nval, 8);
      const uint32_t src = pr.base[i] + static_cast<uint32_t>(cc) * 32u;
      const uint32_t off = src & 15u;
      un[i].lo = st_lds128(src & ~15u);
      un[i].hi = off + 2u * static_cast<uint32_t>(nv) > 16u ? st_lds128((src & ~15u) + 16u) : make_uint4(0u, 0u, 0u, 0u);
      un[i].meta = off | (static_cast<uint32_t>(nv) << 4);
    }
  }
#pragma unroll
  for (int i = 0; i < kStBatch; ++i)
    if ((pr.used >> i) & 1u) st_shared_v4(slot + pr.dst[i], st_extract(un[i]));
}

// KH, KW: the filter's height and width when compiled in (3 x 3: the view
// offsets are computed once and the tap loop is unrolled), 0 for any size.
// RAW: the builders stage each (block, kd)'s input rows and weights in shared
// memory first (st_stage_raw), decode their units once for that pair
// (st_pre_raw) and pack its slots from there (st_pack_pre); otherwise they
// pack straight from global memory (st_build).
template <bool BF16, int KH, int KW, bool RAW>
__global__ void __launch_bounds__(kStThreads, 1) conv_fwd_tc_staged_kernel(const StArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  StTail* tail = reinterpret_cast<StTail*>(smem + a.tail_off);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t smem0 = ptx::smem_u32(smem);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->full[s]), static_cast<uint32_t>(kStBuilders));
      ptx::mbar_init(ptx::smem_u32(&tail->empty[s]), 1u);
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
  if (warp == kStMmaWarp) {
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
  const int kh_n = KH > 0 ? KH : a.kH, kw_n = KW > 0 ? KW : a.kW;
  const int slots_per_tile = a.kD * a.nc16;

  if (RAW && warp < kStBuilderWarps) {
    // ------------------------------------------------------------ builders (raw mode)
    // The builders meet at named barrier 2 twice per (block, kd): before the
    // raw copies overwrite what the previous slots were packed from, and after
    // they landed.  The first meeting also ANDs every builder's status, and
    // only that agreed value ends the loops, so all builders always take the
    // same barriers (a thread whose wait gave up just stops packing).
    const uint32_t raw_x = smem0 + a.raw_x_off, raw_w = smem0 + a.raw_w_off;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true, go = true;
    for (int tile = blockIdx.x; go && tile < a.total_tiles; tile += gridDim.x) {
      const StTile t = st_decode(a, tile);
      for (int kd = 0; kd < a.kD; ++kd) {
        go = named_bar_and(2, kStBuilders, ok);
        if (!go) break;
        st_stage_raw(a, t, kd, raw_x, raw_w, static_cast<int>(threadIdx.x));
        StPre pr;
        st_pre_raw(a, t, kd, raw_x, raw_w, static_cast<int>(threadIdx.x), pr);  // overlaps the copies
        asm volatile("cp.async.wait_all;" ::: "memory");
        named_bar_sync(2, kStBuilders);
        for (int cc = 0; cc < a.nc16; ++cc) {
          if (ok && !wait_bounded(ptx::smem_u32(&tail->empty[s]), ph ^ 1u, abort_flag, a.timeout_ns,
                                  kSiteProducerEmpty))
            ok = false;
          if (ok) {
            st_pack_pre(a, pr, cc, smem0 + static_cast<uint32_t>(s) * a.stage_bytes);
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(ptx::smem_u32(&tail->full[s]));
          }
          if (++s == a.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
  } else if (warp < kStBuilderWarps) {
    // ------------------------------------------------------------ builders
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x) {
      const StTile t = st_decode(a, tile);
      for (int kd = 0; ok && kd < a.kD; ++kd)
        for (int cc = 0; cc < a.nc16; ++cc) {
          if (!wait_bounded(ptx::smem_u32(&tail->empty[s]), ph ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          st_build(a, t, kd, cc, smem0 + static_cast<uint32_t>(s) * a.stage_bytes, static_cast<int>(threadIdx.x));
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(ptx::smem_u32(&tail->full[s]));
          if (++s == a.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
    }
  } else if (warp == kStMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int t = 0;
      if (a.inject_stall)
        ok = wait_bounded(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected);
      // slot 0's weights (K halves 128 bytes apart, 8-row groups 256 apart) and
      // region (K halves one plane apart, N-groups one region row apart)
      const uint64_t dA0 = ptx::smem_desc(smem0, 128u, 256u, 0u);
      const uint64_t dB0 = ptx::smem_desc(smem0 + a.a_bytes, a.plane_bytes, static_cast<uint32_t>(a.Wr) * 16u, 0u);
      const uint64_t slot_off = desc_off(a.stage_bytes);
      uint64_t boff[KH > 0 ? KH * KW : 1];
      if constexpr (KH > 0) {
#pragma unroll
        for (int kh = 0; kh < KH; ++kh)
#pragma unroll
          for (int kw = 0; kw < KW; ++kw)
            boff[kh * KW + kw] = desc_off(static_cast<uint32_t>(kh * a.dh * a.Wr + kw * a.dw) * 16u);
      }
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x, ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag, a.timeout_ns,
                          kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * kStAccStride;
        uint32_t accumulate = 0;
        for (int q = 0; q < slots_per_tile; ++q) {
          if (!wait_bounded(ptx::smem_u32(&tail->full[s]), ph, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint64_t dA = dA0 + static_cast<uint64_t>(s) * slot_off, dB = dB0 + static_cast<uint64_t>(s) * slot_off;
          if constexpr (KH > 0) {
#pragma unroll
            for (int tap = 0; tap < KH * KW; ++tap) {
              ptx::mma_f16(d_tmem, dA + desc_off(static_cast<uint32_t>(tap) * a.tap_bytes), dB + boff[tap], a.idesc,
                           accumulate);
              accumulate = 1;
            }
          } else {
            for (int kh = 0; kh < kh_n; ++kh)
              for (int kw = 0; kw < kw_n; ++kw) {
                const uint32_t tap = static_cast<uint32_t>(kh * kw_n + kw);
                ptx::mma_f16(d_tmem, dA + desc_off(tap * a.tap_bytes),
                             dB + desc_off(static_cast<uint32_t>(kh * a.dh * a.Wr + kw * a.dw) * 16u), a.idesc,
                             accumulate);
                accumulate = 1;
              }
          }
          // the slot is free once these MMAs have read it
          ptx::mma_commit(ptx::smem_u32(&tail->empty[s]));
          if (++s == a.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_u32(&tail->acc_full[acc]));
      }
      // every MMA this thread issued has completed once `drain` fires
      ptx::mma_commit(ptx::smem_u32(&tail->drain));
      wait_drain(ptx::smem_u32(&tail->drain), 0, a.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // warp & 3: tensor-memory lane quarter, output channels 32q .. 32q+31
    const int q = warp & 3;
    const int o = 32 * q + lane;
    const bool any = 32 * q < a.O;  // the same for the whole warp
    uint16_t* __restrict__ y = static_cast<uint16_t*>(a.y);
    const int BP = kStBlockW * a.tile_h;
    int t = 0;
    for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      bool ok = wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                                  kSiteEpiAccFull);
      // the four warps leave together when one of them gave up
      ok = named_bar_and(1, 128, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const StTile tt = st_decode(a, tile);
      const long long plane = (static_cast<long long>(tt.n) * a.Do + tt.od) * a.Ho;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc) * kStAccStride;
      for (int c = 0; any && c < BP; c += 32) {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c), r);
        ptx::tmem_ld_wait();
        const int h0 = tt.h0 + c / kStBlockW;  // 4 output rows of 8 pixels per 32 columns
        if (o < a.O) {
#pragma unroll
          for (int p = 0; p < 32; ++p) {
            const int h = h0 + p / kStBlockW, wo = tt.w0 + (p % kStBlockW);
            if (h < a.Ho && wo < a.Wo)
              y[((plane + h) * a.Wo + wo) * a.O + o] = cvt1<BF16>(__uint_as_float(r[p]));
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&tail->acc_empty[acc]));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kStMmaWarp) ptx::tmem_dealloc(tmem_base, a.tmem_cols);
}

}  // namespace convfwd
