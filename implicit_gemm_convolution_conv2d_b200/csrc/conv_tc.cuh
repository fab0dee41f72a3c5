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
//             zero-fills the halo;  MODE_GATHER: 16 warps compute every
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
constexpr int kMaxTp = 16;  // transposed-convolution phases the gather kernel tracks
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
  kSiteInjected = 6,
};

struct TcArgs {
  int N, D, H, W, C, O;
  int kD, kH, kW;
  int sd, sh, sw, pd, ph, pw, dd, dh, dw;
  // input dilation (gather modes only): input position z of the zero-inserted
  // input holds x[z / id*] when z is a multiple of id*, else 0
  int idil_on, idd, idh, idw;
  int wtrans;         // 1: w is stored [G*Cg][taps][Og] (a transposed convolution's weights)
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
  int kbs;              // K sub-blocks (of kc elements) per pipeline stage
  uint32_t sub_bytes;   // bytes of one sub-block (A and, unless resident, B)
  uint32_t layout_type;  // UMMA smem layout: 2 = 128B swizzle, 4 = 64B, 6 = 32B
  uint32_t sbo;          // bytes between 8-row groups (8 * kc * 2)
  uint32_t idesc;        // tcgen05 instruction descriptor
  uint32_t tmem_cols;
  int rank5;
  int tile_h, tile_w; // halo kernel: output block per CTA (16 x 8)
  int tiles_h, tiles_w;  // halo kernel: blocks per output plane (pair blocks are 2*tile_h high)
  int halo_h, halo_w;    // halo kernel: input block per (channel chunk, kd)
  uint32_t halo_slot_bytes;  // its shared-memory slot (1024-aligned)
  uint32_t halo_bytes;       // bytes one halo load delivers
  int a_slots;               // halo slots in the ring
  int gather_mode;    // GATHER_SCALAR / GATHER_VEC8 / GATHER_SPAN / GATHER_ROWS
  // GATHER_ROWS: input rows of x (viewed as [N*H, W*C]) staged by TMA boxes of
  // one TMA box of stage_rows whole input rows (row_e = W*C elements each,
  // split as n_boxes x box_e so that every box dimension stays <= 256), which
  // lands row after row, row_e elements apart; up to two image segments per tile
  int box_e, n_boxes, stage_rows, row_e;
  uint32_t seg_bytes;   // one segment: stage_rows * row_e * 2, rounded to 128
  uint32_t rows_bytes;  // one buffer: 2 segments
  int Lp;             // span layout: filter-row length kW*C rounded up to 8
  int Kp;             // K as laid out in shared memory (>= K in span layout)
  long long x_elems;  // elements of x (bounds of the unaligned 16-byte loads)
  int mo;             // transposed halo kernel: output channels per tile (MMA M: 64 or 128)
  int b_resident;     // gather: the whole B matrix stays in shared memory
  uint32_t bres_bytes;  // its size (kblocks * BN * 128), 0 when not resident
  int y_tma;          // plain-orientation kernels: the epilogue stores y by TMA tensor stores
  uint32_t epi_bytes; // their staging area (kEpiRowBytes + 1 KB alignment slack), 0 when y_tma is off
  int flip;           // 1: the filter is read reversed in every spatial dimension
  int taps;           // kD*kH*kW
  int w_resident;     // transposed halo kernel: all weight tiles loaded once into stage 0
  int epi_bufs;       // transposed halo kernel: epilogue staging tiles (1 or 2)
  // phase-packed kernel (few input channels): one GEMM row = P output pixels of a row
  int ph_P;            // pixels per GEMM row (P * sw * C is a multiple of 8)
  int ph_ks;           // 16-element K steps per filter row (window of 16 * ph_ks elements)
  int ph_qtot;         // GEMM rows per output row (Wo / P)
  int ph_qint;         // of them, rows whose window lies inside the input row
  int ph_nleft, ph_nright;  // edge rows at the left / right end of an output row
  int ph_rows;         // output rows per tile
  int ph_erow0;        // A-tile row of the first edge row (edge rows use 8-row slots)
  int ph_align;        // GEMM row q's window starts at element P*sw*C*q - ph_align
  uint32_t ph_wbytes;  // bytes of w
  uint32_t ph_bblk;    // one resident B block: N rows x 32 bytes
  uint32_t ph_epi_bytes;  // one epilogue staging tile
  int ph_gcols;        // output columns per epilogue store (64: 128-byte swizzle, 32: 64-byte)
  // transposed convolution by sub-pixel phases (gather kernel, VEC8, Cg % 64
  // == 0): output pixels are grouped by their position modulo the input
  // dilation (the transposed stride); a tile holds pixels of one phase and
  // reads only the taps that reach that phase (the others would multiply the
  // inserted zeros)
  int tp_on;
  int tp_count;                          // phases with at least one output pixel
  int tp_cpt;                            // 64-wide K blocks per tap (Cg / 64)
  int tp_step[3];                        // tap step per dimension: s / gcd(s, d)
  int tp_r[kMaxTp][3];                   // phase residues (output position mod s)
  int tp_A[kMaxTp][3];                   // output extent of the phase per dimension
  int tp_k0[kMaxTp][3], tp_nk[kMaxTp][3];  // first valid tap and valid taps per dimension
  int tp_c0[kMaxTp][3];                  // input offset of the first valid tap: (r - p_lo + k0*d) / s
  int tp_dstep[3];                       // input offset between consecutive valid taps: d / gcd(s, d)
  int tp_tbase[kMaxTp + 1];              // first m tile of each phase
  const void* x;
  const void* w;
  void* y;
  unsigned long long timeout_ns;
  int inject_stall;   // test hook: the MMA thread first waits on a barrier nothing arrives at
};

struct __align__(8) TcSmemTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint64_t stall;     // never arrived on (the injected-timeout test waits here)
  uint64_t bres;      // resident weights loaded
  uint64_t bready;    // phase-packed kernel: both CTAs' halves of B built (leader's)
  uint64_t afull[8];  // halo kernels: input strip slots
  uint64_t aempty[8];
  uint64_t rfull[3];  // row staging (gather): rows of a tile landed
  uint64_t rempty[3]; // row staging: every gather thread is done with the buffer
  int seg_n[3][2];    // row staging, per buffer: image of segment 0 / 1
  int seg_lo[3][2];   // first staged input row of segment 0 / 1
  uint64_t peer_done;   // CTA pairs: the peer's producer finished issuing (leader's)
  uint64_t peer_done_a; // the same for the input-strip ring of the halo kernels
  uint32_t tmem_base;
  volatile int abort_flag;
  volatile int peer_fills;    // CTA pairs: ring fills the peer's producer issued (leader's)
  volatile int peer_fills_a;  // the same for the input-strip ring
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

// CTA-pair producers, after their fill loops: every load either CTA issued
// must have landed before the pair may exit (the loads write the issuing CTA's
// shared memory and signal the leader's barrier).  The leader can see that
// only for ring fills it armed.  So the peer (rank 1) publishes how many fills
// it issued; the leader arms the fills that only the peer issued (with the
// peer's bytes), counts the peer's bytes of fills that only the leader issued
// as done, and waits for the last armed phase of every stage.  A stage is at
// most one phase behind its last armed fill, so one parity wait per stage is
// exact.  peer_bytes(k) gives the peer's bytes of fill k.
template <typename PeerBytes>
__device__ void pair_settle_ring(uint64_t* ring, int nslots, uint64_t* peer_done, volatile int* peer_fills,
                                 bool leader, long long fills, unsigned long long timeout_ns, PeerBytes peer_bytes) {
  if (!leader) {
    ptx::st_shared_cluster_u32(ptx::mapa_shared(ptx::smem_u32(const_cast<int*>(peer_fills)), 0),
                               static_cast<uint32_t>(fills));
    ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(peer_done), 0));
    return;
  }
  const uint32_t pd = ptx::smem_u32(peer_done);
  const uint64_t t0 = ptx::globaltimer_ns();
  bool heard = true;
  while (!ptx::mbar_try_wait_cluster(pd, 0u)) {
    if (ptx::globaltimer_ns() - t0 > timeout_ns) {
      atomicOr(&g_conv_status, 1u | (kSiteDrain << 8));
      heard = false;
      break;
    }
  }
  const long long peer = heard ? static_cast<long long>(static_cast<uint32_t>(*peer_fills)) : fills;
  for (long long k = fills; k < peer; ++k) ptx::mbar_arrive_expect_tx(ptx::smem_u32(&ring[k % nslots]), peer_bytes(k));
  for (long long k = peer; k < fills; ++k) ptx::mbar_complete_tx(ptx::smem_u32(&ring[k % nslots]), peer_bytes(k));
  const long long total = fills > peer ? fills : peer;
  for (int s = 0; s < nslots; ++s) {
    const long long arms = total / nslots + (s < total % nslots ? 1 : 0);
    if (arms > 0) wait_drain(ptx::smem_u32(&ring[s]), static_cast<uint32_t>((arms - 1) & 1), timeout_ns);
  }
}

// The weight / patch ring of a pair kernel (`full`, `stages` slots).
template <typename PeerBytes>
__device__ void pair_settle_ring(TcSmemTail* tail, int stages, bool leader, long long fills,
                                 unsigned long long timeout_ns, PeerBytes peer_bytes) {
  pair_settle_ring(tail->full, stages, &tail->peer_done, &tail->peer_fills, leader, fills, timeout_ns, peer_bytes);
}

struct TileCoord {
  int g, mt, nt;
};

// Transposed-convolution phases: the phase of m tile `mt`, its K-block count,
// its j-th K block, and the output pixel of its local row (false past the
// phase's pixels).
__device__ __forceinline__ int tp_phase(const TcArgs& a, int mt) {
  int ph = 0;
  while (ph + 1 < a.tp_count && mt >= a.tp_tbase[ph + 1]) ++ph;
  return ph;
}
__device__ __forceinline__ int tp_nkb(const TcArgs& a, int ph) {
  return a.tp_nk[ph][0] * a.tp_nk[ph][1] * a.tp_nk[ph][2] * a.tp_cpt;
}
__device__ __forceinline__ int tp_kb(const TcArgs& a, int ph, int j) {
  const int ti = j / a.tp_cpt, chunk = j - (j / a.tp_cpt) * a.tp_cpt;
  const int tw = ti % a.tp_nk[ph][2];
  const int t2 = ti / a.tp_nk[ph][2];
  const int th = t2 % a.tp_nk[ph][1];
  const int td = t2 / a.tp_nk[ph][1];
  const int kd = a.tp_k0[ph][0] + td * a.tp_step[0];
  const int kh = a.tp_k0[ph][1] + th * a.tp_step[1];
  const int kw = a.tp_k0[ph][2] + tw * a.tp_step[2];
  return ((kd * a.kH + kh) * a.kW + kw) * a.tp_cpt + chunk;
}
// Local row of a phase -> image n and the phase-local output position (ad, ah, aw).
__device__ __forceinline__ bool tp_local(const TcArgs& a, int ph, int lrow, int& n, int& ad, int& ah, int& aw) {
  const int Ad = a.tp_A[ph][0], Ah = a.tp_A[ph][1], Aw = a.tp_A[ph][2];
  const unsigned u = static_cast<unsigned>(lrow);
  const unsigned t1 = u / static_cast<unsigned>(Aw);
  const unsigned t2 = t1 / static_cast<unsigned>(Ah);
  const unsigned t3 = t2 / static_cast<unsigned>(Ad);
  n = static_cast<int>(t3);
  aw = static_cast<int>(u - t1 * static_cast<unsigned>(Aw));
  ah = static_cast<int>(t1 - t2 * static_cast<unsigned>(Ah));
  ad = static_cast<int>(t2 - t3 * static_cast<unsigned>(Ad));
  return n < a.N;
}

__device__ __forceinline__ bool tp_pixel(const TcArgs& a, int ph, int lrow, int& n, int& qd, int& qh, int& qw) {
  const int Ad = a.tp_A[ph][0], Ah = a.tp_A[ph][1], Aw = a.tp_A[ph][2];
  const unsigned u = static_cast<unsigned>(lrow);
  const unsigned t1 = u / static_cast<unsigned>(Aw);
  const unsigned t2 = t1 / static_cast<unsigned>(Ah);
  const unsigned t3 = t2 / static_cast<unsigned>(Ad);
  n = static_cast<int>(t3);
  qw = a.tp_r[ph][2] + a.idw * static_cast<int>(u - t1 * static_cast<unsigned>(Aw));
  qh = a.tp_r[ph][1] + a.idh * static_cast<int>(t1 - t2 * static_cast<unsigned>(Ah));
  qd = a.tp_r[ph][0] + a.idd * static_cast<int>(t2 - t3 * static_cast<unsigned>(Ad));
  return n < a.N;
}

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
// 32-bit arithmetic whenever M fits (64-bit division is a long software
// sequence, and every gather thread decodes its pixel once per tile).
__device__ __forceinline__ void decode_pixel(const TcArgs& a, long long m, int& n, int& od, int& oh,
                                             int& ow) {
  if (a.M <= 0x7fffffffLL) {
    const unsigned mm = static_cast<unsigned>(m);
    const unsigned q1 = mm / static_cast<unsigned>(a.Wo);
    const unsigned q2 = q1 / static_cast<unsigned>(a.Ho);
    const unsigned q3 = q2 / static_cast<unsigned>(a.Do);
    ow = static_cast<int>(mm - q1 * static_cast<unsigned>(a.Wo));
    oh = static_cast<int>(q1 - q2 * static_cast<unsigned>(a.Ho));
    od = static_cast<int>(q2 - q3 * static_cast<unsigned>(a.Do));
    n = static_cast<int>(q3);
    return;
  }
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

// Plain-orientation epilogue (accumulator lanes = output pixels, columns =
// output channels): each epilogue warp owns 32 consecutive rows of the tile.
// Per 32-column chunk it writes its rows' 16-bit values into one of its two
// 2 KB staging buffers, [32 rows][64 bytes] in the 64-byte swizzle pattern
// (16-byte chunk j of row r at position j ^ ((r >> 1) & 3), so the 16-byte
// stores of a warp fall in distinct banks), and lane 0 issues one TMA tensor
// store of the [32 x 32] box at (column, first row); rows beyond M are clipped
// by the tensor map.  A buffer is rewritten only after the store issued from
// it two chunks earlier has read it.
constexpr uint32_t kEpiWarpBytes = 4096;   // two 2 KB buffers per epilogue warp
constexpr uint32_t kEpiRowBytes = 4 * kEpiWarpBytes;

template <bool BF16>
__device__ __forceinline__ void epi_store_chunk_tma(uint8_t* warp_bufs, int seq, const uint32_t (&r)[32],
                                                    const CUtensorMap* tmap_y, int col, long long row0) {
  const int lane = threadIdx.x & 31;
  uint8_t* buf = warp_bufs + (seq & 1) * 2048;
  if (lane == 0) ptx::bulk_wait_group_read<1>();
  __syncwarp();
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 v;
    v.x = pack2<BF16>(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
    v.y = pack2<BF16>(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
    v.z = pack2<BF16>(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
    v.w = pack2<BF16>(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ sw) << 4)) = v;
  }
  ptx::fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    ptx::tma_store_2d(tmap_y, ptx::smem_u32(buf), col, static_cast<int32_t>(row0));
    ptx::bulk_commit_group();
  }
}


// ----------------------------------------------------------------------------
// MMA issue.  One thread issues every tcgen05.mma of a CTA, and on B200 the
// instruction stream around the MMAs decides whether the tensor pipe stays
// fed: a per-instruction rebuild of the operand descriptors in a loop with a
// run-time trip count cost ~220 SM cycles per 128x256x16 MMA in a probe,
// against 128 (the pipe's own rate) for fully unrolled issue of descriptors
// that only advance by constants.  So descriptors are built once, moved by
// 64-bit adds (the start address is bits 0..13 in 16-byte units, and shared
// memory is below 256 KB, so an add never carries out of the field), and the
// K steps of one sub-block are issued by an unrolled compile-time loop.
// ----------------------------------------------------------------------------

// Descriptor address units (16 bytes) for a byte offset.
__device__ __forceinline__ uint64_t desc_off(uint32_t bytes) { return static_cast<uint64_t>(bytes >> 4); }

// KS MMAs of K = 16 over one sub-block: both operands advance 32 bytes
// (2 descriptor units) per step.  acc0 = 0 overwrites the accumulator with
// the first product.
template <int KS, bool PAIR>
__device__ __forceinline__ void mma_ksteps(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc0) {
#pragma unroll
  for (int k = 0; k < KS; ++k) {
    if constexpr (PAIR) ptx::mma_f16_pair(d_tmem, da + 2 * k, db + 2 * k, idesc, k == 0 ? acc0 : 1u);
    else ptx::mma_f16(d_tmem, da + 2 * k, db + 2 * k, idesc, k == 0 ? acc0 : 1u);
  }
}

// Filter tap (kd*kH + kh)*kW + kw of the weights that input tap `tap` multiplies:
// itself, or with flip the tap mirrored in every spatial dimension, which in
// this numbering is taps - 1 - tap.
__device__ __forceinline__ int wtap(const TcArgs& a, int tap) { return a.flip ? a.taps - 1 - tap : tap; }

// The same for a run-time step count of 1 to 4 (channel chunks of 64, 32 or
// 16 elements; 3 for a 48-element phase-packed window).
template <bool PAIR>
__device__ __forceinline__ void mma_sub(int ksteps, uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t idesc,
                                        uint32_t acc0) {
  if (ksteps == 4) mma_ksteps<4, PAIR>(d_tmem, da, db, idesc, acc0);
  else if (ksteps == 3) mma_ksteps<3, PAIR>(d_tmem, da, db, idesc, acc0);
  else if (ksteps == 2) mma_ksteps<2, PAIR>(d_tmem, da, db, idesc, acc0);
  else mma_ksteps<1, PAIR>(d_tmem, da, db, idesc, acc0);
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
  static constexpr int kProducerWarps = 16;
};

template <int MODE>
constexpr int tc_threads() {
  return (TcRoles<MODE>::kProducerWarps + 1 + 4) * 32;
}

// ----------------------------------------------------------------------------
// Gather producer: 512 threads (16 warps) fill one stage with zero fill.
// Thread t owns A row t % 128 and the 16-element quarter t / 128 of every
// 64-wide K block; element k of a row is (kd, kh, kw, c) in weight order (or
// the span layout).  B is either resident (loaded once per CTA) or gathered
// per stage.
// ----------------------------------------------------------------------------
struct GatherRow {
  bool valid;
  long long nbase;  // element offset of x[n, 0, 0, 0, g*Cg]
  int id0, ih0, iw0;
  int jlo, jhi;     // span mode: valid offsets within a filter row
  uint32_t rseg;    // row staging: byte address of this pixel's image segment
  int lr0;          // row staging: staged row of input row ih0 in that segment
};

// Position in the span layout of K: element j of filter row (kd, kh).  Each
// gather thread walks it in steps of 8 instead of dividing k by Lp per call.
struct SpanPos {
  int j, kh, kd;
};

__device__ __forceinline__ void span_step8(const TcArgs& a, SpanPos& p) {
  p.j += 8;
  if (p.j == a.Lp) {
    p.j = 0;
    if (++p.kh == a.kH) {
      p.kh = 0;
      ++p.kd;
    }
  }
}

__device__ __forceinline__ SpanPos span_pos(const TcArgs& a, int k) {
  const int span = k / a.Lp;
  SpanPos p;
  p.j = k - span * a.Lp;
  p.kh = span % a.kH;
  p.kd = span / a.kH;
  return p;
}

// Position z of an input dimension dilated by s (zeros inserted between
// elements): true, with z replaced by the element index, when z is a multiple
// of s inside the input of n elements.
__device__ __forceinline__ bool undilate(int& z, int s, int n) {
  if (z < 0 || z % s != 0) return false;
  z /= s;
  return z < n;
}

// One filter row (kd, kh) of one output pixel: offset of x[n, id, ih, 0, g*Cg]
// and whether that input row exists.
template <bool TR = false>
__device__ __forceinline__ bool gather_span(const TcArgs& a, const GatherRow& st, int kd, int kh,
                                            long long& rowptr) {
  int id = st.id0 + kd * a.dd;
  int ih = st.ih0 + kh * a.dh;
  bool ok;
  if (TR && a.idil_on) {
    ok = st.valid && kd < a.kD && undilate(id, a.idd, a.D) && undilate(ih, a.idh, a.H);
  } else {
    ok = st.valid && kd < a.kD && static_cast<unsigned>(id) < static_cast<unsigned>(a.D) &&
         static_cast<unsigned>(ih) < static_cast<unsigned>(a.H);
  }
  if (TR) {
    rowptr = st.nbase + (static_cast<long long>(ok ? id : 0) * a.H + (ok ? ih : 0)) * static_cast<long long>(a.W) * a.C;
  } else {
    rowptr = st.nbase + (static_cast<long long>(id) * a.H + ih) * static_cast<long long>(a.W) * a.C;
  }
  return ok;
}

// Input column of one tap: the element index (in place) and whether it exists.
template <bool TR = false>
__device__ __forceinline__ bool gather_col(const TcArgs& a, int& iw) {
  if (TR && a.idil_on) return undilate(iw, a.idw, a.W);
  return static_cast<unsigned>(iw) < static_cast<unsigned>(a.W);
}

__device__ __forceinline__ void store_chunk(uint8_t* a_tile, int r, int ch, uint4 v) {
  *reinterpret_cast<uint4*>(a_tile + sw128_offset(r, ch)) = v;
}

// Scalar gather of the 8 elements p[e] for e in [e_lo, e_hi), zeros elsewhere.
__device__ __forceinline__ uint4 load8_masked(const uint16_t* p, int e_lo, int e_hi) {
  uint32_t v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = (e >= e_lo && e < e_hi) ? __ldg(p + e) : 0u;
  return make_uint4(v[0] | (v[1] << 16), v[2] | (v[3] << 16), v[4] | (v[5] << 16), v[6] | (v[7] << 16));
}

// NCH 8-element chunks (K elements k0 .. k0+8*NCH-1) of one A row.
//
// GATHER_VEC8 (C/G % 8 == 0): a chunk is 8 channels of one input pixel, one
// aligned 16-byte load, or zeros when the pixel is in the padding.
// GATHER_SPAN (one group, dilation_w == 1): K is laid out per filter row
// (kd, kh) as the kW*C contiguous elements of that row, zero-padded to Lp (a
// multiple of 8), so a chunk never crosses a row; element j of row (kd, kh) is
// x[n, id, ih, iw0, 0] + j and exists for j in [jlo, jhi).
// GATHER_SCALAR: element-wise (kw, c) walk with its own bounds check.
enum { GATHER_SCALAR = 0, GATHER_VEC8 = 1, GATHER_SPAN = 2, GATHER_ROWS = 3 };

template <int NCH, bool TR = false>
__device__ __forceinline__ void gather_a_vec8(const TcArgs& a, const GatherRow& st, int k0, uint8_t* a_tile,
                                              int r, int chunk0) {
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  const int tap = k0 / a.Cg;
  int c = k0 - tap * a.Cg;
  int kw = tap % a.kW;
  const int t2 = tap / a.kW;
  int kh = t2 % a.kH;
  int kd = t2 / a.kH;
  long long rowptr;
  bool rok = gather_span<TR>(a, st, kd, kh, rowptr);
  uint4 v[NCH];
#pragma unroll
  for (int q = 0; q < NCH; ++q) {
    int iw = st.iw0 + kw * a.dw;
    v[q] = make_uint4(0, 0, 0, 0);
    if (rok && gather_col<TR>(a, iw))
      v[q] = __ldg(reinterpret_cast<const uint4*>(x + rowptr + static_cast<long long>(iw) * a.C + c));
    c += 8;
    if (c == a.Cg) {
      c = 0;
      if (++kw == a.kW) {
        kw = 0;
        if (++kh == a.kH) {
          kh = 0;
          ++kd;
        }
        rok = gather_span<TR>(a, st, kd, kh, rowptr);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < NCH; ++q) store_chunk(a_tile, r, chunk0 + q, v[q]);
}

// Halfwords h .. h+7 of the 16 halfwords in (b0, b1), h in 0..7.
__device__ __forceinline__ uint4 extract8(const uint4& b0, const uint4& b1, unsigned h) {
  const uint32_t w[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
  const unsigned sh = h >> 1;
  uint32_t u[5];
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const uint32_t lo = (sh & 1) ? w[(k + 1) & 7] : w[k];
    const uint32_t hi = (sh & 1) ? w[(k + 3) & 7] : w[(k + 2) & 7];
    u[k] = (sh & 2) ? hi : lo;  // w[k + sh]
  }
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] = (h & 1) ? __funnelshift_r(u[i], u[i + 1], 16) : u[i];
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// Zero the halfwords of v whose bit in the 8-bit mask is clear.
__device__ __forceinline__ uint4 mask8(uint4 v, unsigned m) {
  const auto keep = [m](int i) -> uint32_t {
    return ((m >> (2 * i)) & 1 ? 0x0000FFFFu : 0u) | ((m >> (2 * i + 1)) & 1 ? 0xFFFF0000u : 0u);
  };
  v.x &= keep(0);
  v.y &= keep(1);
  v.z &= keep(2);
  v.w &= keep(3);
  return v;
}

// The loads of gather_a_span, issued apart from their use so that other work
// (the B chunks of the same K block) can run while they are in flight.
template <int NCH>
struct SpanLoads {
  uint4 b0[NCH], b1[NCH];
  unsigned hsh[NCH], msk[NCH];
};

template <int NCH>
__device__ __forceinline__ void gather_a_span_issue(const TcArgs& a, const GatherRow& st, SpanPos& pos,
                                                    SpanLoads<NCH>& L) {
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  int j = pos.j, kh = pos.kh, kd = pos.kd;
  long long rowptr;
  bool rok = gather_span(a, st, kd, kh, rowptr);
  rowptr += static_cast<long long>(st.iw0) * a.C;
  // every load of the NCH chunks: aligned 16-byte blocks that cover the chunk
  // (the halo and the row ends are masked when the chunks are stored)
#pragma unroll
  for (int q = 0; q < NCH; ++q) {
    L.b0[q] = make_uint4(0, 0, 0, 0);
    L.b1[q] = make_uint4(0, 0, 0, 0);
    L.hsh[q] = 0;
    L.msk[q] = 0;
    if (rok && j + 8 > st.jlo && j < st.jhi) {
      const int lo = max(st.jlo - j, 0), hi = min(st.jhi - j, 8);
      const long long e0 = rowptr + j;
      const long long a0 = e0 & ~7LL;
      if (a0 >= 0 && a0 + 16 <= a.x_elems) {
        L.hsh[q] = static_cast<unsigned>(e0 - a0);
        L.msk[q] = ((1u << hi) - 1u) & ~((1u << lo) - 1u);
        L.b0[q] = __ldg(reinterpret_cast<const uint4*>(x + a0));
        if (L.hsh[q] != 0) L.b1[q] = __ldg(reinterpret_cast<const uint4*>(x + a0 + 8));
      } else {
        L.b0[q] = load8_masked(x + e0, lo, hi);  // at the tensor's ends: element loads
        L.msk[q] = 0xFFu;
      }
    }
    j += 8;
    if (j == a.Lp) {
      j = 0;
      if (++kh == a.kH) {
        kh = 0;
        ++kd;
      }
      rok = gather_span(a, st, kd, kh, rowptr);
      rowptr += static_cast<long long>(st.iw0) * a.C;
    }
  }
  pos.j = j;
  pos.kh = kh;
  pos.kd = kd;
}

// Shift the loaded blocks into place, mask, store.
template <int NCH>
__device__ __forceinline__ void gather_a_span_store(const SpanLoads<NCH>& L, uint8_t* a_tile, int r, int chunk0) {
#pragma unroll
  for (int q = 0; q < NCH; ++q) store_chunk(a_tile, r, chunk0 + q, mask8(extract8(L.b0[q], L.b1[q], L.hsh[q]), L.msk[q]));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// GATHER_ROWS: the same span layout as gather_a_span, read from the input
// rows staged in shared memory.  `rows` is the staging buffer of this tile,
// seg_n / seg_lo its segments (image, first staged input row).  A chunk that
// lies wholly inside the row is five aligned 32-bit loads shifted into place
// (its first element may be odd); chunks at the image edge take element loads.
template <int NCH>
__device__ __forceinline__ void gather_a_rows(const TcArgs& a, const GatherRow& st, SpanPos& pos, uint8_t* a_tile,
                                              int r, int chunk0) {
  int j = pos.j, kh = pos.kh;
  const bool in_k = pos.kd < a.kD;  // false in the zero padding after the last filter row
  // byte address of the staged row holding filter row kh of this output pixel (or none)
  const auto row_base = [&](int khh, bool& ok) -> uint32_t {
    const int ih = st.ih0 + khh * a.dh;
    const int lr = st.lr0 + khh * a.dh;
    ok = st.valid && in_k && khh < a.kH && static_cast<unsigned>(ih) < static_cast<unsigned>(a.H) &&
         static_cast<unsigned>(lr) < static_cast<unsigned>(a.stage_rows);
    return st.rseg + static_cast<uint32_t>(lr) * static_cast<uint32_t>(a.row_e) * 2u;
  };
  bool rok;
  uint32_t rb = row_base(kh, rok);
  const int ebase = st.iw0 * a.C;  // element of x[n, ih, iw0, 0] within the row (may be negative)
  uint4 v[NCH];
#pragma unroll
  for (int q = 0; q < NCH; ++q) {
    v[q] = make_uint4(0, 0, 0, 0);
    if (rok && j + 8 > st.jlo && j < st.jhi) {
      if (j >= st.jlo && j + 8 <= st.jhi) {
        // all eight elements exist: element e0 >= 0
        const int e0 = ebase + j;
        const uint32_t addr = rb + static_cast<uint32_t>(e0 & ~1) * 2u;
        const uint32_t sh = static_cast<uint32_t>(e0 & 1) * 16u;
        const uint32_t w0 = lds32(addr), w1 = lds32(addr + 4), w2 = lds32(addr + 8), w3 = lds32(addr + 12),
                       w4 = lds32(addr + 16);
        v[q] = make_uint4(__funnelshift_r(w0, w1, sh), __funnelshift_r(w1, w2, sh), __funnelshift_r(w2, w3, sh),
                          __funnelshift_r(w3, w4, sh));
      } else {
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int jj = j + i;
          h[i] = (jj >= st.jlo && jj < st.jhi) ? lds16(rb + static_cast<uint32_t>(ebase + jj) * 2u) : 0u;
        }
        v[q] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
      }
    }
    j += 8;
    if (j == a.Lp) {
      j = 0;
      ++kh;
      rb = row_base(kh, rok);
    }
  }
  pos.j = j;
  pos.kh = kh;
#pragma unroll
  for (int q = 0; q < NCH; ++q) store_chunk(a_tile, r, chunk0 + q, v[q]);
}

template <int NCH, bool TR = false>
__device__ __forceinline__ void gather_a_scalar(const TcArgs& a, const GatherRow& st, int k0, uint8_t* a_tile,
                                                int r, int chunk0) {
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  uint32_t v[8 * NCH];
  const int tap = k0 / a.Cg;
  int c = k0 - tap * a.Cg;
  int kw = tap % a.kW;
  const int t2 = tap / a.kW;
  int kh = t2 % a.kH;
  int kd = t2 / a.kH;
  long long rowptr;
  bool ok = gather_span<TR>(a, st, kd, kh, rowptr);
#pragma unroll
  for (int e = 0; e < 8 * NCH; ++e) {
    int iw = st.iw0 + kw * a.dw;
    v[e] = (ok && gather_col<TR>(a, iw)) ? __ldg(x + rowptr + static_cast<long long>(iw) * a.C + c) : 0u;
    if (++c == a.Cg) {
      c = 0;
      if (++kw == a.kW) {
        kw = 0;
        if (++kh == a.kH) {
          kh = 0;
          ++kd;
        }
        ok = gather_span<TR>(a, st, kd, kh, rowptr);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < NCH; ++q)
    store_chunk(a_tile, r, chunk0 + q,
                make_uint4(v[8 * q] | (v[8 * q + 1] << 16), v[8 * q + 2] | (v[8 * q + 3] << 16),
                           v[8 * q + 4] | (v[8 * q + 5] << 16), v[8 * q + 6] | (v[8 * q + 7] << 16)));
}

// Sub-pixel phase tiles of a transposed convolution: the j-th K block of
// phase ph is 64 channels of one valid tap, whose input pixel is the row's
// phase-local position (held in st.id0/ih0/iw0) plus the tap's offset, with
// no division; NCH 16-byte chunks of that pixel.
template <int NCH>
__device__ __forceinline__ void gather_a_tp(const TcArgs& a, const GatherRow& st, int ph, int j, uint8_t* a_tile,
                                            int r, int chunk0) {
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(a.x);
  const int ti = j / a.tp_cpt;
  const int cblk = j - ti * a.tp_cpt;
  const int tw = ti % a.tp_nk[ph][2];
  const int t2 = ti / a.tp_nk[ph][2];
  const int th = t2 % a.tp_nk[ph][1];
  const int td = t2 / a.tp_nk[ph][1];
  const int id = st.id0 + a.tp_c0[ph][0] + td * a.tp_dstep[0];
  const int ih = st.ih0 + a.tp_c0[ph][1] + th * a.tp_dstep[1];
  const int iw = st.iw0 + a.tp_c0[ph][2] + tw * a.tp_dstep[2];
  const bool ok = st.valid && static_cast<unsigned>(id) < static_cast<unsigned>(a.D) &&
                  static_cast<unsigned>(ih) < static_cast<unsigned>(a.H) &&
                  static_cast<unsigned>(iw) < static_cast<unsigned>(a.W);
  const long long p = st.nbase + ((static_cast<long long>(ok ? id : 0) * a.H + (ok ? ih : 0)) * a.W + (ok ? iw : 0)) *
                                     static_cast<long long>(a.C) +
                      cblk * 64 + chunk0 * 8;
#pragma unroll
  for (int q = 0; q < NCH; ++q) {
    const uint4 v = ok ? __ldg(reinterpret_cast<const uint4*>(x + p + q * 8)) : make_uint4(0, 0, 0, 0);
    store_chunk(a_tile, r, chunk0 + q, v);
  }
}

// B rows [0, BN) x K elements [kbase, kbase+64) of group g, output channels
// starting at n0, into a swizzled BN x 128-byte tile.  `nthreads` threads
// share the 8*BN chunks.  In span layout, padded K element kp of filter row
// s = kp / Lp, offset j = kp % Lp, is w[o, s*kW*C + j] for j < kW*C, else 0.
template <bool TR = false>
__device__ __forceinline__ void gather_b_block(const TcArgs& a, int g, int n0, int kbase, uint8_t* b_tile,
                                               int tid, int nthreads) {
  const uint16_t* __restrict__ w = static_cast<const uint16_t*>(a.w);
  if (TR && a.wtrans && (a.Cg & 7) == 0 && (a.Og & 7) == 0) {
    // Transposed weights [G*Cg][taps][Og], 8-aligned channel counts: a thread
    // takes 8 B rows (output channels) x one 8-element K chunk (8 channels c of
    // one tap); the 8 channels' rows of 8 output channels are 16-byte loads,
    // transposed in registers into the 8 rows' chunks.
#pragma unroll 1
    for (int q = tid; q < a.BN; q += nthreads) {
      const int rg = q >> 3, ch = q & 7;
      const int oc0 = n0 + rg * 8;
      const int kp0 = kbase + ch * 8;
      uint32_t in[8][4];
      if (oc0 < a.Og && kp0 < a.K) {
        const int tap = kp0 / a.Cg;
        const int c0 = kp0 - tap * a.Cg;
        const long long base = (static_cast<long long>(g * a.Cg + c0) * a.taps + wtap(a, tap)) * a.Og + oc0;
        const long long pitch = static_cast<long long>(a.taps) * a.Og;  // between consecutive channels c
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(w + base + e * pitch));
          in[e][0] = v.x; in[e][1] = v.y; in[e][2] = v.z; in[e][3] = v.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) in[e][0] = in[e][1] = in[e][2] = in[e][3] = 0u;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        // row r (output channel oc0 + r): halfword r of each channel's vector
        const uint32_t sel = (r & 1) ? 0x7632u : 0x5410u;
        uint4 o;
        o.x = __byte_perm(in[0][r >> 1], in[1][r >> 1], sel);
        o.y = __byte_perm(in[2][r >> 1], in[3][r >> 1], sel);
        o.z = __byte_perm(in[4][r >> 1], in[5][r >> 1], sel);
        o.w = __byte_perm(in[6][r >> 1], in[7][r >> 1], sel);
        *reinterpret_cast<uint4*>(b_tile + sw128_offset(rg * 8 + r, ch)) = o;
      }
    }
    return;
  }
  const bool span_layout = a.gather_mode == GATHER_SPAN || a.gather_mode == GATHER_ROWS;
  const bool vec = (a.K & 7) == 0 && !span_layout;
  const int L = a.kW * a.C;
#pragma unroll 1
  for (int q = tid; q < a.BN * 8; q += nthreads) {
    const int o = q >> 3, ch = q & 7;
    const int oc = n0 + o;
    const int kp0 = kbase + ch * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (oc < a.Og && kp0 < a.Kp) {
      const long long rowoff = static_cast<long long>(g * a.Og + oc) * a.K;
      if (TR && a.wtrans) {
        // w stored [G*Cg][taps][Og]: K element k = tap*Cg + c of output
        // channel oc multiplies w[g*Cg + c][tap (mirrored under flip)][oc]
        uint16_t e8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int k = kp0 + e;
          const int tap = k / a.Cg;
          const long long wi =
              (static_cast<long long>(g * a.Cg + (k - tap * a.Cg)) * a.taps + wtap(a, tap)) * a.Og + oc;
          e8[e] = k < a.K ? w[wi] : uint16_t(0);
        }
        v = *reinterpret_cast<const uint4*>(e8);
      } else if (span_layout) {  // (never with flip: the planner uses the other layouts)
        // the 8 elements at w[o, sp*kW*C + j0 ...] (those past the filter row's
        // kW*C are zero): two aligned 16-byte loads shifted into place
        const int sp = kp0 / a.Lp;
        const int j0 = kp0 - sp * a.Lp;
        const int cnt = min(8, L - j0);
        if (cnt > 0) {
          const long long e0 = rowoff + static_cast<long long>(sp) * L + j0;
          const long long a0 = e0 & ~7LL;
          if (a0 + 16 <= static_cast<long long>(a.O) * a.K) {
            const unsigned h = static_cast<unsigned>(e0 - a0);
            const uint4 b0 = __ldg(reinterpret_cast<const uint4*>(w + a0));
            const uint4 b1 = h != 0 ? __ldg(reinterpret_cast<const uint4*>(w + a0 + 8)) : make_uint4(0, 0, 0, 0);
            v = mask8(extract8(b0, b1, h), (1u << cnt) - 1u);
          } else {
            v = load8_masked(w + e0, 0, cnt);  // at the tensor's end: element loads
          }
        }
      } else if (a.flip) {
        // K element k = tap*Cg + c multiplies w[o, taps-1-tap, c]
        uint16_t e8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int k = kp0 + e;
          const int tap = k / a.Cg;
          e8[e] = k < a.K ? w[rowoff + static_cast<long long>(wtap(a, tap)) * a.Cg + (k - tap * a.Cg)] : uint16_t(0);
        }
        v = *reinterpret_cast<const uint4*>(e8);
      } else if (vec) {
        v = __ldg(reinterpret_cast<const uint4*>(w + rowoff + kp0));
      } else {
        v = load8_masked(w + rowoff + kp0, 0, a.K - kp0);
      }
    }
    *reinterpret_cast<uint4*>(b_tile + sw128_offset(o, ch)) = v;
  }
}

// GATHER_ROWS: stage the input rows one 128-row output tile reads.  The tile's
// pixels lie in at most two images (host guarantees Ho*Wo >= 128); for each
// image segment the contiguous range of input rows its filter rows touch is
// loaded as one 3-D TMA box (box_e x n_boxes x stage_rows) from x viewed as
// [N*H][row_e / box_e][box_e]
// viewed as [N*H, W*C] (zero fill beyond the tensor).  Issued by one thread.
__device__ __forceinline__ void issue_rows(const TcArgs& a, const CUtensorMap* tmap, TcSmemTail* tail, uint8_t* rowsbuf,
                                           int tile, int b) {
  const TileCoord tc = decode_tile(a, tile);
  const long long m0 = static_cast<long long>(tc.mt) * kBM;
  const long long m1 = min(m0 + kBM - 1, a.M - 1);
  int n0, od, oh0, ow, n1, oh1;
  decode_pixel(a, m0, n0, od, oh0, ow);
  decode_pixel(a, m1, n1, od, oh1, ow);
  const int segn[2] = {n0, n1 != n0 ? n1 : -1};
  const int ohf[2] = {oh0, 0};
  const int ohl[2] = {n1 != n0 ? a.Ho - 1 : oh1, oh1};
  const uint32_t box_bytes = static_cast<uint32_t>(a.stage_rows) * static_cast<uint32_t>(a.row_e) * 2u;
  int lo[2] = {0, 0};
  bool load[2] = {false, false};
  uint32_t bytes = 0;
  for (int sg = 0; sg < 2; ++sg) {
    if (segn[sg] < 0) continue;
    const int ih_lo = max(0, ohf[sg] * a.sh - a.ph);
    const int ih_hi = min(a.H - 1, ohl[sg] * a.sh - a.ph + (a.kH - 1) * a.dh);
    lo[sg] = ih_lo;
    load[sg] = ih_hi >= ih_lo;
    if (load[sg]) bytes += box_bytes;
  }
  tail->seg_n[b][0] = segn[0];
  tail->seg_n[b][1] = segn[1];
  tail->seg_lo[b][0] = lo[0];
  tail->seg_lo[b][1] = lo[1];
  const uint32_t fb = ptx::smem_u32(&tail->rfull[b]);
  ptx::mbar_arrive_expect_tx(fb, bytes);  // release: the segment table above is published with it
  for (int sg = 0; sg < 2; ++sg) {
    if (!load[sg]) continue;
    ptx::tma_load_3d(ptx::smem_u32(rowsbuf + b * a.rows_bytes + sg * a.seg_bytes), tmap, fb, 0, 0,
                     segn[sg] * a.H + lo[sg]);
  }
}

// ----------------------------------------------------------------------------
// The kernel.
// ----------------------------------------------------------------------------
// TR: the transposed-convolution gather (input dilation, transposed weights);
// TP: with sub-pixel phases.  Separate instantiations, so that the forward
// gather kernel keeps its registers.
template <int MODE, bool BF16, bool TR = false, bool TP = false>
__global__ void __launch_bounds__(tc_threads<MODE>(), 1)
    conv_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_y, const TcArgs a) {
  constexpr int kProdWarps = TcRoles<MODE>::kProducerWarps;
  constexpr int kMmaWarp = kProdWarps;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* bres = smem + a.stages * a.stage_bytes;  // resident B (gather mode), 1024-aligned
  uint8_t* rowsbuf = bres + a.bres_bytes;            // staged input rows (GATHER_ROWS), 3 buffers
  uint8_t* epi_area = rowsbuf + 3 * a.rows_bytes;    // epilogue staging (y_tma), with 1 KB of slack
  uint8_t* epibuf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(epi_area) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(epi_area + a.epi_bytes);
  constexpr uint32_t kProdThreads = kProdWarps * 32;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      ptx::mbar_init(ptx::smem_u32(&tail->full[s]), MODE == MODE_TMA ? 1u : kProdThreads);
      ptx::mbar_init(ptx::smem_u32(&tail->empty[s]), 1u);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_u32(&tail->acc_full[b]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->acc_empty[b]), 4u);
    }
    ptx::mbar_init(ptx::smem_u32(&tail->drain), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->stall), 1u);
    ptx::mbar_init(ptx::smem_u32(&tail->bres), kProdThreads);
    for (int b = 0; b < 3; ++b) {
      ptx::mbar_init(ptx::smem_u32(&tail->rfull[b]), 1u);
      ptx::mbar_init(ptx::smem_u32(&tail->rempty[b]), kProdThreads);
    }
    tail->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (threadIdx.x == 32 && (MODE == MODE_TMA || a.gather_mode == GATHER_ROWS)) {
    ptx::prefetch_tmap(&tmap_x);
    if (MODE == MODE_TMA) ptx::prefetch_tmap(&tmap_w);
  }
  if (warp == kMmaWarp) {
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
          for (int kb = 0; kb < a.kblocks; kb += a.kbs) {
            const int nsub = min(a.kbs, a.kblocks - kb);
            if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag,
                              a.timeout_ns, kSiteProducerEmpty)) {
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
              ptx::tma_load_2d(sb, &tmap_w, fb, wtap(a, tap) * a.Cg + cchunk * a.kc, orow);
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
              wait_drain(ptx::smem_u32(&tail->full[s]), static_cast<uint32_t>((arms - 1) & 1),
                         a.timeout_ns);
          }
        }
      }
      __syncwarp();
    } else {
      const int tid = threadIdx.x;  // 0 .. kProdThreads-1
      const int r = tid & 127;      // A row
      // which 16 of the 64 K elements of every K block this thread builds
      // (16 producer warps: enough threads in flight to hide each chunk's
      // dependent address, load and shift chain)
      constexpr int kParts = kProdThreads / kBM;
      constexpr int kNch = 8 / kParts;  // 8-element chunks per thread per K block
      const int part = tid >> 7;
      if (a.b_resident) {
        // the whole B matrix, once per CTA: [kblock][BN rows][128 B]
        for (int kb = 0; kb < a.kblocks; ++kb)
          gather_b_block<TR>(a, 0, 0, kb * 64, bres + static_cast<uint32_t>(kb) * a.BN * 128u, tid,
                         kProdThreads);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(ptx::smem_u32(&tail->bres));
      }
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const bool rows_mode = a.gather_mode == GATHER_ROWS;
      int lt = 0;  // local tile counter; row-staging buffer lt % 3, its use lt / 3
      for (int tile = blockIdx.x; ok && tile < a.total_tiles; tile += gridDim.x, ++lt) {
        const TileCoord tc = decode_tile(a, tile);
        const int rb = lt % 3;
        if (rows_mode &&
            !wait_bounded(ptx::smem_u32(&tail->rfull[rb]), static_cast<uint32_t>((lt / 3) & 1), abort_flag,
                          a.timeout_ns, kSiteProducerEmpty)) {
          ok = false;
          break;
        }
        GatherRow st;
        int n = 0, od = 0, oh = 0, ow = 0;
        int tph = 0, nkb = a.kblocks;
        if constexpr (TP) {
          // od, oh, ow: the phase-local output position (input offsets are added per tap)
          tph = tp_phase(a, tc.mt);
          nkb = tp_nkb(a, tph);
          st.valid = tp_local(a, tph, (tc.mt - a.tp_tbase[tph]) * kBM + r, n, od, oh, ow);
          if (!st.valid) n = od = oh = ow = 0;
        } else {
          const long long m = static_cast<long long>(tc.mt) * kBM + r;
          st.valid = m < a.M;
          if (st.valid) decode_pixel(a, m, n, od, oh, ow);
        }
        st.nbase = static_cast<long long>(n) * a.D * a.H * a.W * a.C + static_cast<long long>(tc.g) * a.Cg;
        if constexpr (TP) {
          st.id0 = od;
          st.ih0 = oh;
          st.iw0 = ow;
        } else {
          st.id0 = od * a.sd - a.pd;
          st.ih0 = oh * a.sh - a.ph;
          st.iw0 = ow * a.sw - a.pw;
        }
        st.jlo = max(0, -st.iw0) * a.C;
        st.jhi = min(a.kW, a.W - st.iw0) * a.C;
        if (st.jhi < st.jlo) st.jhi = st.jlo;
        if (rows_mode) {
          const int seg = (n == tail->seg_n[rb][0]) ? 0 : 1;
          st.rseg = ptx::smem_u32(rowsbuf + rb * a.rows_bytes) + static_cast<uint32_t>(seg) * a.seg_bytes;
          st.lr0 = st.ih0 - tail->seg_lo[rb][seg];
        }
        // this thread's first K element of every 64-wide K block
        SpanPos pos = span_pos(a, part * kNch * 8);
        const int n0 = tc.nt * a.BN;
        for (int kb = 0; kb < nkb; kb += a.kbs) {
          const int nsub = min(a.kbs, nkb - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          for (int j = 0; j < nsub; ++j) {
            uint8_t* sa = smem + stage * a.stage_bytes + j * a.sub_bytes;
            const int kbm = TP ? tp_kb(a, tph, kb + j) : kb + j;  // the K block loaded
            const int k0 = kbm * 64 + part * kNch * 8;
            if (TP)
              gather_a_tp<kNch>(a, st, tph, kb + j, sa, r, part * kNch);
            else if (a.gather_mode == GATHER_VEC8)
              gather_a_vec8<kNch, TR>(a, st, k0, sa, r, part * kNch);
            else if (rows_mode) {
              gather_a_rows<kNch>(a, st, pos, sa, r, part * kNch);
              // skip the other threads' chunks of this K block
              for (int i = 0; i < 8 - kNch; ++i) span_step8(a, pos);
            } else if (a.gather_mode == GATHER_SPAN) {
              // the A loads are in flight while this thread gathers its share of B
              SpanLoads<kNch> sl;
              gather_a_span_issue<kNch>(a, st, pos, sl);
              for (int i = 0; i < 8 - kNch; ++i) span_step8(a, pos);
              if (!a.b_resident) gather_b_block<TR>(a, tc.g, n0, kbm * 64, sa + a.a_bytes, tid, kProdThreads);
              gather_a_span_store<kNch>(sl, sa, r, part * kNch);
              continue;
            } else
              gather_a_scalar<kNch, TR>(a, st, k0, sa, r, part * kNch);
            if (!a.b_resident) gather_b_block<TR>(a, tc.g, n0, kbm * 64, sa + a.a_bytes, tid, kProdThreads);
          }
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(ptx::smem_u32(&tail->full[stage]));
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        // this thread is done reading the tile's staged rows
        if (rows_mode && ok) ptx::mbar_arrive(ptx::smem_u32(&tail->rempty[rb]));
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ row loader (GATHER_ROWS)
    if (MODE == MODE_GATHER && a.gather_mode == GATHER_ROWS && lane == 1) {
      int lt = 0;
      for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++lt) {
        const int rb = lt % 3, use = lt / 3;
        if (use >= 1 && !wait_bounded(ptx::smem_u32(&tail->rempty[rb]), static_cast<uint32_t>((use - 1) & 1),
                                      abort_flag, a.timeout_ns, kSiteProducerEmpty))
          break;
        issue_rows(a, &tmap_x, tail, rowsbuf, tile, rb);
      }
      // before the CTA can exit, every row load issued must have landed
      for (int b = 0; b < 3 && b < lt; ++b) {
        const int last_use = (lt - 1 - b) / 3;  // uses of buffer b: tiles b, b+3, ... < lt
        wait_drain(ptx::smem_u32(&tail->rfull[b]), static_cast<uint32_t>(last_use & 1), a.timeout_ns);
      }
    }
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int t = 0;
      if (a.inject_stall)
        ok = wait_bounded(ptx::smem_u32(&tail->stall), 0u, abort_flag, a.timeout_ns, kSiteInjected);
      if (ok && a.b_resident)
        ok = wait_bounded(ptx::smem_u32(&tail->bres), 0u, abort_flag, a.timeout_ns, kSiteMmaFull);
      // descriptors built once; moved by constant offsets below
      const uint64_t d_ring = ptx::smem_desc(ptx::smem_u32(smem), 16, a.sbo, a.layout_type);
      const uint64_t d_res = ptx::smem_desc(ptx::smem_u32(bres), 16, a.sbo, a.layout_type);
      const uint64_t a_off = desc_off(a.a_bytes), sub_off = desc_off(a.sub_bytes), st_off = desc_off(a.stage_bytes);
      const uint64_t res_step = desc_off(static_cast<uint32_t>(a.BN) * 128u);
      const int ksteps = a.kc >> 4;
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
        int tph = 0, nkb = a.kblocks;
        if constexpr (TP) {
          tph = tp_phase(a, decode_tile(a, tile).mt);
          nkb = tp_nkb(a, tph);  // 0: no tap reaches the phase, the epilogue writes zeros
        }
        for (int kb = 0; kb < nkb; kb += a.kbs) {
          const int nsub = min(a.kbs, nkb - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns,
                            kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          uint64_t da = d_ring + static_cast<uint64_t>(stage) * st_off;
          for (int j = 0; j < nsub; ++j) {
            const int kbm = TP ? tp_kb(a, tph, kb + j) : kb + j;
            const uint64_t db = a.b_resident ? d_res + static_cast<uint64_t>(kbm) * res_step : da + a_off;
            mma_sub<false>(ksteps, d_tmem, da, db, a.idesc, (kb + j) != 0 ? 1u : 0u);
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
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = q * 32 + lane;
    uint16_t* __restrict__ y = static_cast<uint16_t*>(a.y);
    int t = 0, epi_seq = 0;
    for (int tile = blockIdx.x; tile < a.total_tiles; tile += gridDim.x, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      if (!wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag,
                             a.timeout_ns, kSiteEpiAccFull))
        break;
      ptx::tc_fence_after();
      const TileCoord tc = decode_tile(a, tile);
      long long m = static_cast<long long>(tc.mt) * kBM + row;
      bool mvalid = m < a.M;
      bool zero = false;  // a phase no tap reaches: its outputs are 0
      if constexpr (TP) {
        const int tph = tp_phase(a, tc.mt);
        int n, qd, qh, qw;
        mvalid = tp_pixel(a, tph, (tc.mt - a.tp_tbase[tph]) * kBM + row, n, qd, qh, qw);
        m = mvalid ? ((static_cast<long long>(n) * a.Do + qd) * a.Ho + qh) * a.Wo + qw : 0;
        zero = tp_nkb(a, tph) == 0;
      }
      const int n0 = tc.nt * a.BN;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * a.BN);
      if (!TP && a.y_tma) {
        // staged TMA stores of this warp's 32 rows (never the phase tiles, whose rows are not consecutive)
        const long long row0 = static_cast<long long>(tc.mt) * kBM + q * 32;
        const int ncols = row0 < a.M ? min(a.BN, a.Og - n0) : 0;  // no store starts past the last row
        for (int c = 0; c < ncols; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld_32x32b_x32(taddr + c, r);
          ptx::tmem_ld_wait();
          epi_store_chunk_tma<BF16>(epibuf + q * kEpiWarpBytes, epi_seq++, r, &tmap_y, tc.g * a.Og + n0 + c, row0);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&tail->acc_empty[acc]));
        continue;
      }
      const long long ybase = m * a.O + static_cast<long long>(tc.g) * a.Og;
      for (int c = 0; c < a.BN; c += 32) {
        uint32_t r[32];
        if (zero) {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;  // +0.0f
        } else {
          ptx::tmem_ld_32x32b_x32(taddr + c, r);
          ptx::tmem_ld_wait();
        }
        const int col0 = n0 + c;
        const int nvalid = min(32, a.Og - col0);
        if (mvalid && nvalid > 0) {
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
    // every tensor store has read its buffer and written y before exit
    if (lane == 0 && a.y_tma) ptx::bulk_wait_group<0>();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem_base, a.tmem_cols);
}

}  // namespace convfwd

namespace convfwd {

// ----------------------------------------------------------------------------
// CTA-pair variant of the TMA kernel: a cluster of two CTAs on two SMs owns a
// 256 x BN output tile and issues tcgen05.mma.cta_group::2 (M = 256).  Each CTA
// loads its own 128 rows of A and its own BN/2 rows of B, so per K stage a CTA
// pulls half the weight bytes of a 128 x BN single-CTA tile for the same MMA
// work.  Both CTAs' TMA loads complete on the leader's (rank 0) `full`
// barrier; the leader's single MMA thread issues for the pair and its commits
// arrive on `empty` / `acc_full` in both CTAs; each CTA's epilogue drains its
// own 128 accumulator rows and arrives on the leader's `acc_empty`.
// ----------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(192, 1)
    conv_fwd_tc_pair_kernel(const __grid_constant__ CUtensorMap tmap_x,
                            const __grid_constant__ CUtensorMap tmap_w,
                            const __grid_constant__ CUtensorMap tmap_y, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* epi_area = smem + a.stages * a.stage_bytes;  // epilogue staging (y_tma), with 1 KB of slack
  uint8_t* epibuf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(epi_area) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
  TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(epi_area + a.epi_bytes);
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
        const TileCoord tc = decode_tile(a, tile);
        int n, od, oh, ow;
        decode_pixel(a, static_cast<long long>(tc.mt) * (2 * kBM) + rank * kBM, n, od, oh, ow);
        const int cw = ow * a.sw - a.pw, chh = oh * a.sh - a.ph, cd = od * a.sd - a.pd;
        const int brow = tc.g * a.Og + tc.nt * a.BN + static_cast<int>(rank) * half_bn;
        int tap = 0, cchunk = 0;
        for (int kb = 0; kb < a.kblocks; kb += a.kbs) {
          const int nsub = min(a.kbs, a.kblocks - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->empty[stage]), phase ^ 1u, abort_flag, a.timeout_ns,
                            kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = ptx::smem_u32(&tail->full[stage]);
          if (leader)
            ptx::mbar_arrive_expect_tx(fb_local, 2u * static_cast<uint32_t>(nsub) * (a.a_bytes + a.b_bytes));
          const uint32_t fb = ptx::mapa_shared(fb_local, 0);
          for (int j = 0; j < nsub; ++j) {
            const uint32_t sa = ptx::smem_u32(smem + stage * a.stage_bytes + j * a.sub_bytes);
            const uint32_t sb = sa + a.a_bytes;
            const int kw = tap % a.kW;
            const int kh = (tap / a.kW) % a.kH;
            const int kd = tap / (a.kW * a.kH);
            const int c0 = tc.g * a.Cg + cchunk * a.kc;
            if (a.rank5)
              ptx::tma_load_im2col_5d_pair(sa, &tmap_x, fb, c0, cw, chh, cd, n, static_cast<uint16_t>(kw * a.dw),
                                           static_cast<uint16_t>(kh * a.dh), static_cast<uint16_t>(kd * a.dd));
            else
              ptx::tma_load_im2col_4d_pair(sa, &tmap_x, fb, c0, cw, chh, n, static_cast<uint16_t>(kw * a.dw),
                                           static_cast<uint16_t>(kh * a.dh));
            ptx::tma_load_2d_pair(sb, &tmap_w, fb, wtap(a, tap) * a.Cg + cchunk * a.kc, brow);
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
      // fill k of a tile's sequence carries nsub = min(kbs, kblocks - j*kbs) sub-blocks, j = k mod fills per tile
      const int fpt = (a.kblocks + a.kbs - 1) / a.kbs;
      pair_settle_ring(tail, a.stages, leader, fills, a.timeout_ns, [&](long long k) {
        const int j = static_cast<int>(k % fpt);
        return static_cast<uint32_t>(min(a.kbs, a.kblocks - j * a.kbs)) * (a.a_bytes + a.b_bytes);
      });
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
      // descriptors built once; moved by constant offsets below
      const uint64_t d_ring = ptx::smem_desc(ptx::smem_u32(smem), 16, a.sbo, a.layout_type);
      const uint64_t a_off = desc_off(a.a_bytes), sub_off = desc_off(a.sub_bytes), st_off = desc_off(a.stage_bytes);
      const int ksteps = a.kc >> 4;
      for (int tile = pair; ok && tile < a.total_tiles; tile += npairs, ++t) {
        const int acc = t & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
        if (!wait_bounded(ptx::smem_u32(&tail->acc_empty[acc]), acc_phase ^ 1u, abort_flag, a.timeout_ns,
                          kSiteMmaAccEmpty)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        for (int kb = 0; kb < a.kblocks; kb += a.kbs) {
          const int nsub = min(a.kbs, a.kblocks - kb);
          if (!wait_bounded(ptx::smem_u32(&tail->full[stage]), phase, abort_flag, a.timeout_ns, kSiteMmaFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          uint64_t da = d_ring + static_cast<uint64_t>(stage) * st_off;
          for (int j = 0; j < nsub; ++j) {
            mma_sub<true>(ksteps, d_tmem, da, da + a_off, a.idesc, (kb + j) != 0 ? 1u : 0u);
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
    const int row = q * 32 + lane;
    uint16_t* __restrict__ y = static_cast<uint16_t*>(a.y);
    int t = 0, epi_seq = 0;
    for (int tile = pair; tile < a.total_tiles; tile += npairs, ++t) {
      const int acc = t & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(t >> 1) & 1u;
      if (!wait_bounded_warp(ptx::smem_u32(&tail->acc_full[acc]), acc_phase, abort_flag, a.timeout_ns,
                             kSiteEpiAccFull))
        break;
      ptx::tc_fence_after();
      const TileCoord tc = decode_tile(a, tile);
      const long long m = static_cast<long long>(tc.mt) * (2 * kBM) + rank * kBM + row;
      const int n0 = tc.nt * a.BN;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
      if (a.y_tma) {
        // staged TMA stores of this warp's 32 rows
        const long long row0 = static_cast<long long>(tc.mt) * (2 * kBM) + rank * kBM + q * 32;
        const int ncols = row0 < a.M ? min(a.BN, a.Og - n0) : 0;  // no store starts past the last row
        for (int c = 0; c < ncols; c += 32) {
          uint32_t r[32];
          ptx::tmem_ld_32x32b_x32(taddr + c, r);
          ptx::tmem_ld_wait();
          epi_store_chunk_tma<BF16>(epibuf + q * kEpiWarpBytes, epi_seq++, r, &tmap_y, tc.g * a.Og + n0 + c, row0);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(&tail->acc_empty[acc]), 0));
        continue;
      }
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
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(&tail->acc_empty[acc]), 0));
    }
    // every tensor store has read its buffer and written y before exit
    if (lane == 0 && a.y_tma) ptx::bulk_wait_group<0>();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the leader's MMAs (which read this CTA's smem) are complete
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc_pair(tmem_base, a.tmem_cols);
}

}  // namespace convfwd
