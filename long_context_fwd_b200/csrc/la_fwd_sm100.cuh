// la_fwd_sm100.cuh -- Lightning Attention prefill on B200 tensor cores (tcgen05).
//
// Operation ("MiniMax-M1" model entry (archdb), linear/SSM layer field:
// per-head exponential decay, 128x128 state per head; positional field: decay
// only, no RoPE; "MiniMax-01" (redeep.blog), "What Makes 1M Context Hard":
// linear-complexity attention), per (b, h) sequence with gamma = exp(-lambda_h):
//     o_t = sum_{s <= t} gamma^(t-s) (q_t . k_s) v_s
//
// Blocked form.  The sequence is cut into blocks of 128 tokens; for a block
// with local rows i, j, length len and the state S before it (D x E, fp32):
//   Sc   = Q K^T                                   (tensor cores, fp32 in TMEM)
//   P_ij = Sc_ij gamma^(i-j) for j <= i, else 0    (CUDA cores, bf16 back to TMEM)
//   O    = (gamma^(i+1) Q) S_bf16 + P V             (tensor cores, one accumulator)
//   S   <- gamma^len S + (gamma^(len-1-j) K)^T V   (tensor cores, fp32 in TMEM)
// Every decay factor used is gamma^m with 0 <= m <= 128, so nothing overflows.
//
// Work splits (the items of each CTA are computed in la_schedule.cuh):
//   * whole sequences, or a balanced hand-over when B*H >= SMs (a sequence cut
//     between two CTAs: the first part publishes its final state, the second
//     part runs last and starts from it);
//   * the split scan when SMs/8 <= B*H < SMs (a local-state pass over the first
//     parts of all sequences, cut into pieces; a share that starts inside a
//     sequence adds up the pieces before it);
//   * the chunked scan otherwise.  Work item w = chunk * (B*H) + seq.  A chunk
//     with a successor first computes its local state A_c = sum_j
//     gamma^(Lc-1-j) k_j^T v_j over its tokens (phase 1, K/V kept in L2 with an
//     evict-last hint), then takes the inclusive state of the previous chunk
//     from global memory (spin on a flag, bounded in time), publishes its own
//     inclusive state gamma^Lc S_prev + A_c, and runs the blocked form from
//     S_prev (phase 2).  Items are handed out through an atomic ticket, so every
//     chunk's predecessor is held by a CTA that is already running: no
//     co-residency assumption.
// Published states are 64 KiB fp32 in scratch with a 64-bit flag stored with
// release semantics; the hand-over and the split scan publish a value unique
// to the launch, so their flags need no clearing between launches.
//
// Roles (448 threads, one CTA per SM):
//   warps 0..7   group X: decay-causal mask of Q K^T into P (bf16, TMEM),
//                gamma^(i+1) Q into TMEM, decayed K in place in shared memory.
//                Thread t owns TMEM lane / tile row r = 32 (warp % 4) + lane and
//                the column half hf = warp / 4.
//   warps 8..11  group Y: the state's bf16 copy and decay, the chunk scan, and
//                the epilogue (TMEM -> swizzled shared memory -> TMA store).
//                Thread t owns row r = 32 (warp % 4) + lane, all 128 columns.
//   warp 12      TMA producer: Q/K/V tiles into three 2-slot rings.
//   warp 13      TMEM allocator and single-thread tcgen05.mma issuer: per block
//                the state update, inter and intra products, then the next
//                block's Q K^T (which waits for the next K tile).
// X and Y run concurrently on different blocks' data.
// TMEM (512 columns): S/P double buffer [0,256), O [256,384), state [384,512).
// After group X has read the scores of an S buffer it rewrites the buffer with
// two bf16 operands for the MMAs that follow: P (columns j < 64 in [0,32), j >= 64
// in [64,96)) and gamma^(i+1) Q (d < 64 in [32,64), d >= 64 in [96,128)).  Each
// thread overwrites only columns it has read itself.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "la_schedule.cuh"
#include "sm100_ptx.cuh"

namespace la {
namespace fwd {

// BLK (tokens per block = MMA M) and HD (D = E) come from la_schedule.cuh.
constexpr int X_THREADS = 256;
constexpr int Y_THREADS = 128;
constexpr int X_WARPS = X_THREADS / 32;
constexpr int Y_WARPS = Y_THREADS / 32;
constexpr int X_WARP0 = 0;
constexpr int Y_WARP0 = 8;
constexpr int PRODUCER_WARP = 12;
constexpr int MMA_WARP = 13;
constexpr int THREADS = 448;

constexpr uint32_t PLANE = 16384;       // 128 rows x 128 B
constexpr uint32_t TILE = 2 * PLANE;    // 128 x 128 bf16
constexpr uint32_t OFF_Q = 0;           // 2 slots
constexpr uint32_t OFF_K = 2 * TILE;    // 2 slots
constexpr uint32_t OFF_V = 4 * TILE;    // 2 slots
constexpr uint32_t OFF_KVB = 6 * TILE;  // bf16 copy of the state (MMA B operand)
constexpr uint32_t OFF_BAR = 7 * TILE;
constexpr uint32_t OFF_GTAB = OFF_BAR + 512;  // 256 floats: gtab[u] = gamma^(127-u), 0 for u > 127
constexpr uint32_t OFF_MISC = OFF_GTAB + 1024;
// split scan: the pieces an entering state chains, (slot, blocks from the
// piece's end to the share's start) pairs written by group Y's leader.  The
// host takes the split only for at least SMs/8 sequences, so a chain holds
// at most G/nseq + G2/nseq + 3 <= 19 pieces.
constexpr int CHAIN_MAX = 32;
constexpr uint32_t OFF_CHAIN = OFF_MISC + 128;
constexpr uint32_t SMEM_USED = OFF_CHAIN + 8 * CHAIN_MAX;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227u * 1024u, "dynamic shared memory above the per-CTA limit");

constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_KV = 384;

// Phase 1 reads only K and V.  It lays a 3-deep ring of (K, V) pairs over the
// Q/K/V ring memory (pair slot p = [p * 2 TILE, +2 TILE): K then V), so three
// blocks are in flight instead of two.  Pair slot p overlaps phase-2 ring p
// (0: Q, 1: K, 2: V); the producer hands memory over between the two layouts.
constexpr int P1_SLOTS = 3;
__host__ __device__ constexpr uint32_t p1_base(uint32_t slot) { return OFF_Q + slot * 2u * TILE; }

enum BarId : int {
  B_QF = 0, B_QE = 2, B_KF = 4, B_KE = 6, B_VF = 8, B_VE = 10,
  B_SF = 12, B_SE = 14,
  B_READY = 16, B_KVB_READY, B_KVO_DONE, B_O_FULL, B_O_EMPTY, B_AGG_FULL, B_KV_FREE,
  B_WF = 24, B_WE = 26,
  B_XSYNC = 28, B_YSYNC = 29, B_DRAIN = 30,
  B_P1F = 32,  // phase 1: K/V pair loaded, one per pair slot (3)
  B_P1E = 35,  // phase 1: pair slot free again (3)
  B_KT = 38,   // phase 1: decayed K tile of a pair slot ready (3)
  B_ACT = 41,  // fused layer: Q and K tiles of a block activated (2)
  B_CHAIN = 43,      // split scan: the entering chain listed and its pieces published
  B_CHAIN_DONE = 44, // split scan: group X has combined the entering state
  B_COUNT = 45
};

// Optional event trace (compiled only with -DLA_TRACE): %globaltimer stamps of
// each role's pipeline events for the first few CTAs, for timeline analysis.
#ifdef LA_TRACE
constexpr int TRACE_CTAS = 4, TRACE_EVENTS = 28, TRACE_SLOTS = 256;
__device__ unsigned long long* g_trace;
__device__ __forceinline__ void trace_event(int ev, uint32_t idx) {
  if (g_trace && blockIdx.x < TRACE_CTAS && idx < TRACE_SLOTS)
    g_trace[(blockIdx.x * TRACE_EVENTS + ev) * TRACE_SLOTS + idx] = globaltimer_ns();
}
#define LA_TRACE_EVENT(ev, idx) trace_event((ev), (idx))
#else
#define LA_TRACE_EVENT(ev, idx) ((void)0)
#endif

// A paired launch runs two operators on alternate CTAs: the schedule sees a
// grid of half the CTAs, and each role has its own scratch and output.
__device__ __forceinline__ int cta_role(const Params& p) {
  return p.paired ? static_cast<int>(blockIdx.x & 1u) : 0;
}
__device__ __forceinline__ int vgrid(const Params& p) {
  return static_cast<int>(gridDim.x >> (p.paired ? 1 : 0));
}
__device__ __forceinline__ int vcta(const Params& p) {
  return static_cast<int>(blockIdx.x >> (p.paired ? 1 : 0));
}

// Work item for work index w on this CTA.
__device__ __forceinline__ bool get_item(const Params& p, const volatile uint32_t* m, int w,
                                         Item& it) {
  return get_item(p, vgrid(p), vcta(p), m, w, it);
}

__device__ __forceinline__ void st_release_gpu(unsigned long long* ptr, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(ptr), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long* ptr) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ptr) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// Shared-memory access with explicit state-space instructions
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ float lds32f(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts32f(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t x, float f) {
  return pack_bf16x2(bf16lo_to_f32(x) * f, bf16hi_to_f32(x) * f);
}

// sigmoid(x) = (1 + tanh(x / 2)) / 2 from the hardware tanh (tanh.approx.f32,
// one MUFU operation per element): the fused layer's gate.
__device__ __forceinline__ float tanh_hw(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_hw(float x) { return fmaf(0.5f, tanh_hw(0.5f * x), 0.5f); }

// f * SiLU of a bf16 pair, f x sigmoid(x), in fp32 and rounded once (one MUFU
// operation per element).  Packed bf16 arithmetic with the bf16 tanh was
// tried: its error reached 7% on heads with fast decay, where few tokens
// average it out, so it is not used.
__device__ __forceinline__ uint32_t silu_scale_bf16x2(uint32_t x, float f) {
  const float lo = bf16lo_to_f32(x), hi = bf16hi_to_f32(x);
  const float hl = 0.5f * lo, hh = 0.5f * hi;
  const float fl = f * hl, fh = f * hh;
  return pack_bf16x2(fmaf(fl, tanh_hw(hl), fl), fmaf(fh, tanh_hw(hh), fh));
}

// f * SiLU of the 64 bf16 of one 128-byte swizzled row, in place (the fused
// layer's activation of q, k and v as they arrive in shared memory).
__device__ __forceinline__ void silu_row(uint32_t rowaddr, uint32_t row, float f) {
  uint4 x[8];
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) x[c] = lds128(rowaddr + ((c ^ (row & 7u)) << 4));
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) {
    x[c].x = silu_scale_bf16x2(x[c].x, f);
    x[c].y = silu_scale_bf16x2(x[c].y, f);
    x[c].z = silu_scale_bf16x2(x[c].z, f);
    x[c].w = silu_scale_bf16x2(x[c].w, f);
  }
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) sts128(rowaddr + ((c ^ (row & 7u)) << 4), x[c]);
}

// Multiplies the 64 bf16 of one 128-byte swizzled row by f, in place.  All 8
// loads are issued before any store; the physical chunk order (c ^ row) keeps
// 8 consecutive rows on distinct banks.
__device__ __forceinline__ void scale_row(uint32_t rowaddr, uint32_t row, float f) {
  uint4 x[8];
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) x[c] = lds128(rowaddr + ((c ^ (row & 7u)) << 4));
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) {
    x[c].x = scale_bf16x2(x[c].x, f);
    x[c].y = scale_bf16x2(x[c].y, f);
    x[c].z = scale_bf16x2(x[c].z, f);
    x[c].w = scale_bf16x2(x[c].w, f);
  }
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) sts128(rowaddr + ((c ^ (row & 7u)) << 4), x[c]);
}

// Writes 32 floats (times f) as bf16 into logical chunks [4*h, 4*h+4) of a
// 128-byte swizzled row (logical chunk c holds row elements 8c..8c+7).
__device__ __forceinline__ void store_half_bf16(uint32_t rowaddr, uint32_t row, uint32_t h,
                                                const uint32_t (&x)[32], float f) {
#pragma unroll
  for (uint32_t c = 0; c < 4; ++c) {
    uint4 u;
    u.x = pack_bf16x2(__uint_as_float(x[8 * c + 0]) * f, __uint_as_float(x[8 * c + 1]) * f);
    u.y = pack_bf16x2(__uint_as_float(x[8 * c + 2]) * f, __uint_as_float(x[8 * c + 3]) * f);
    u.z = pack_bf16x2(__uint_as_float(x[8 * c + 4]) * f, __uint_as_float(x[8 * c + 5]) * f);
    u.w = pack_bf16x2(__uint_as_float(x[8 * c + 6]) * f, __uint_as_float(x[8 * c + 7]) * f);
    sts128(rowaddr + (((4 * h + c) ^ (row & 7u)) << 4), u);
  }
}

// Writes 32 floats into one 128-byte swizzled fp32 row (logical chunk c holds
// elements 4c..4c+3).
__device__ __forceinline__ void store_row_f32(uint32_t rowaddr, uint32_t row,
                                              const uint32_t (&x)[32]) {
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c)
    sts128(rowaddr + ((c ^ (row & 7u)) << 4),
           make_uint4(x[4 * c + 0], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]));
}

__device__ __forceinline__ void tmem_st32_scaled(uint32_t taddr, const uint32_t (&x)[32], float f) {
  uint32_t a[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(x[i]) * f);
  tmem_st32(taddr, a);
}

// ---------------------------------------------------------------------------
// Context, failure handling, bounded waits
// ---------------------------------------------------------------------------
struct Ctx {
  uint8_t* sm;
  uint32_t sbase;           // shared-space address of sm
  uint64_t* bar;
  volatile uint32_t* misc;  // [0] TMEM base, [1..2] work slots, [3] abort,
                            // [4..17] this CTA's share of a static split,
                            // [18] length of the chain below
  volatile uint32_t* chain;  // CHAIN_MAX (slot, distance) pairs
  uint32_t tmem;
};

__device__ __forceinline__ bool aborted(const Ctx& c) { return c.misc[3] != 0; }

__device__ __forceinline__ void fail(const Ctx& c, const Params& p, int code) {
  c.misc[3] = 1;
  atomicOr(p.status, code);
}

// Bounded wait (single-thread roles); on time-out records the failure.
__device__ __forceinline__ bool wait_bar(const Ctx& c, const Params& p, int id, uint32_t parity) {
  if (aborted(c)) return false;
  if (mbar_wait(&c.bar[id], parity, p.wait_limit_ns)) return true;
  fail(c, p, 1);
  return false;
}

// Warp-uniform bounded wait for the compute groups: all 32 lanes take the same
// branch, so the warp-collective tcgen05.ld/st that follow are never split.
__device__ __forceinline__ bool cwait(const Ctx& c, const Params& p, int id, uint32_t parity) {
  bool ok = !aborted(c) && mbar_wait(&c.bar[id], parity, p.wait_limit_ns);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && lane_id() == 0) fail(c, p, 1);
  return ok;
}

// One arrival per warp once every lane has reached this point (the barriers
// the compute groups signal count warps, not threads).
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if (lane_id() == 0) mbar_arrive(bar);
}

// Synchronises the threads of one compute group through an mbarrier
// (bounded, unlike bar.sync, so a failed wait elsewhere cannot hang the group).
__device__ __forceinline__ bool gsync(const Ctx& c, const Params& p, int id, uint32_t& n) {
  warp_arrive(&c.bar[id]);
  return cwait(c, p, id, n++ & 1u);
}

// Next work index: this CTA's item count in the static splits, a dynamic ticket
// for chunked runs, a static stride otherwise (n counts this CTA's items).
__device__ __forceinline__ int next_work(const Params& p, int& n) {
  if (p.mode != MODE_TICKETS) return n++;
  if (p.nchunks > 1) return p.ticket_base + atomicAdd(cta_role(p) ? p.ticket1 : p.ticket, 1);
  return vcta(p) + vgrid(p) * n++;
}

// Coordinates (beyond the column) of a tile of tokens [row, row + 128) of
// head hh of batch bb in a 4-D tensor map whose outer dimensions are ordered
// as `slots` says (see make_tmap_4d).
struct TmaCoords {
  int c1, c2, c3;
};
__device__ __forceinline__ TmaCoords tma_coords(int slots, int row, int hh, int bb) {
  const int st = slots & 3, sh = (slots >> 2) & 3;
  TmaCoords c;
  c.c1 = st == 1 ? row : sh == 1 ? hh : bb;
  c.c2 = st == 2 ? row : sh == 2 ? hh : bb;
  c.c3 = st == 3 ? row : sh == 3 ? hh : bb;
  return c;
}

// One 64-column half of a tile of 128 tokens of sequence seq (= bb * H + hh):
// contiguous head-major tensors use 3-D maps [B*H][N][cols]; strided ones 4-D
// maps (measured: the 4-D form costs a few percent, so it is only used when
// the layout needs it).
template <int RANK>
__device__ __forceinline__ void tile_load(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                          int row, int seq, int hh, int bb, int slots,
                                          uint64_t pol) {
  if constexpr (RANK == 3) {
    tma_load_3d(dst, map, bar, x, row, seq, pol);
  } else {
    const TmaCoords tc = tma_coords(slots, row, hh, bb);
    tma_load_4d(dst, map, bar, x, tc.c1, tc.c2, tc.c3, pol);
  }
}

template <int RANK>
__device__ __forceinline__ void tile_store(const CUtensorMap* map, const void* src, int x, int row,
                                           int seq, int hh, int bb, int slots, uint64_t pol) {
  if constexpr (RANK == 3) {
    tma_store_3d(map, src, x, row, seq, pol);
  } else {
    const TmaCoords tc = tma_coords(slots, row, hh, bb);
    tma_store_4d(map, src, x, tc.c1, tc.c2, tc.c3, pol);
  }
}

// ---------------------------------------------------------------------------
// Producer: one thread issues every TMA load.
// ---------------------------------------------------------------------------
// REV (anti-causal runs): work items and blocks are in reversed token order
// tau = N - 1 - t; the tile of tau-block [tb, tb + 128) is tokens
// [N - tb - 128, N - tb), loaded in increasing token order (a negative start
// row reads zeros), so a tile row r holds local reversed index 127 - r.
__device__ __forceinline__ int tile_row(const Params& p, int tb, bool rev) {
  return rev ? p.N - tb - BLK : tb;
}

template <int RANK, bool REV>
__device__ void producer(const Ctx& c, const Params& p, const CUtensorMap* tq,
                         const CUtensorMap* tk, const CUtensorMap* tv) {
  const uint64_t pol_first = policy_evict_first();
  const uint64_t pol_last = policy_evict_last();
  uint32_t q_it = 0, k_it = 0, v_it = 0, w_it = 0;
  int n_items = 0;
  auto load = [&](int ring_f, int ring_e, uint32_t off, uint32_t& it, const CUtensorMap* tm,
                  int tensor, int row, int seq, int hh, int bb, uint64_t pol) -> bool {
    const uint32_t s = it & 1u;
    if (it >= 2 && !wait_bar(c, p, ring_e + s, ((it >> 1) - 1) & 1u)) return false;
    uint8_t* dst = c.sm + off + s * TILE;
    LA_TRACE_EVENT(ring_f == B_QF ? 0 : ring_f == B_KF ? 1 : 2, it);
    mbar_arrive_expect_tx(&c.bar[ring_f + s], TILE);
    tile_load<RANK>(dst, tm, &c.bar[ring_f + s], 0, row, seq, hh, bb, p.cslot[tensor], pol);
    tile_load<RANK>(dst + PLANE, tm, &c.bar[ring_f + s], 64, row, seq, hh, bb, p.cslot[tensor],
                    pol);
    ++it;
    return true;
  };
  // Before leaving, wait (bounded) for every load still in flight so no TMA
  // write lands in shared memory after the CTA exits.
  auto drain_ring = [&](int ring_f, uint32_t n) {
    for (uint32_t j = n >= 2 ? n - 2 : 0; j < n; ++j)
      mbar_wait(&c.bar[ring_f + (j & 1u)], (j >> 1) & 1u, p.wait_limit_ns);
  };
  auto drain = [&]() {
    drain_ring(B_QF, q_it);
    drain_ring(B_KF, k_it);
    drain_ring(B_VF, v_it);
  };
  uint32_t p1_it = 0;          // phase-1 pair loads issued
  bool pairs_pending = false;  // pairs issued since the last pairs_released()
  // Waits until the phase-2 ring overlapping pair slot `slot` has released its
  // last two tiles (their phases have completed, so these waits do not alias).
  auto ring_released = [&](uint32_t slot) -> bool {
    const int e = slot == 0 ? B_QE : slot == 1 ? B_KE : B_VE;
    const uint32_t n = slot == 0 ? q_it : slot == 1 ? k_it : v_it;
    for (uint32_t j = n >= 2 ? n - 2 : 0; j < n; ++j)
      if (!wait_bar(c, p, e + (j & 1u), (j >> 1) & 1u)) return false;
    return true;
  };
  // Waits until every phase-1 pair issued so far has been consumed.
  auto pairs_released = [&]() -> bool {
    for (uint32_t j = p1_it >= P1_SLOTS ? p1_it - P1_SLOTS : 0; j < p1_it; ++j)
      if (!wait_bar(c, p, B_P1E + (j % P1_SLOTS), (j / P1_SLOTS) & 1u)) return false;
    return true;
  };
  for (;;) {
    const int w = next_work(p, n_items);
    const uint32_t ws = w_it & 1u;
    if (w_it >= 2 && !wait_bar(c, p, B_WE + ws, ((w_it >> 1) - 1) & 1u)) break;
    c.misc[1 + ws] = static_cast<uint32_t>(w);
    mbar_arrive(&c.bar[B_WF + ws]);
    ++w_it;
    Item it;
    if (!get_item(p, c.misc, w, it)) break;
    const int hh = it.seq % p.H, bb = it.seq / p.H;
    bool ok = true;
    if (it.phase1) {
      for (int b = 0; b < it.nb && ok; ++b) {
        const uint32_t slot = p1_it % P1_SLOTS, use = p1_it / P1_SLOTS;
        if (b < P1_SLOTS) ok = ring_released(slot);  // first use in this item
        if (ok && use >= 1) ok = wait_bar(c, p, B_P1E + slot, (use - 1) & 1u);
        if (!ok) break;
        const int row = tile_row(p, it.t0 + b * BLK, REV);
        uint8_t* dst = c.sm + p1_base(slot);
        uint64_t* full = &c.bar[B_P1F + slot];
        mbar_arrive_expect_tx(full, 2 * TILE);
        tile_load<RANK>(dst, tk, full, 0, row, it.seq, hh, bb, p.cslot[1], pol_last);
        tile_load<RANK>(dst + PLANE, tk, full, 64, row, it.seq, hh, bb, p.cslot[1], pol_last);
        tile_load<RANK>(dst + TILE, tv, full, 0, row, it.seq, hh, bb, p.cslot[2], pol_last);
        tile_load<RANK>(dst + TILE + PLANE, tv, full, 64, row, it.seq, hh, bb, p.cslot[2],
                        pol_last);
        ++p1_it;
        pairs_pending = true;
      }
    }
    if (ok && it.p2 && pairs_pending) {  // phase-2 tiles reuse the pairs' memory
      ok = pairs_released();
      pairs_pending = false;
    }
    for (int n = 0; n < (it.p2 ? it.nb : 0) && ok; ++n) {
      const int row = tile_row(p, it.t0 + n * BLK, REV);
      ok = load(B_QF, B_QE, OFF_Q, q_it, tq, 0, row, it.seq, hh, bb, pol_first) &&
           load(B_KF, B_KE, OFF_K, k_it, tk, 1, row, it.seq, hh, bb, pol_first) &&
           load(B_VF, B_VE, OFF_V, v_it, tv, 2, row, it.seq, hh, bb, pol_first);
    }
    if (!ok) break;
  }
  for (uint32_t j = p1_it >= P1_SLOTS ? p1_it - P1_SLOTS : 0; j < p1_it; ++j)
    mbar_wait(&c.bar[B_P1F + (j % P1_SLOTS)], (j / P1_SLOTS) & 1u, p.wait_limit_ns);
  drain();
}

// ---------------------------------------------------------------------------
// MMA issuer: one thread issues every tcgen05.mma.
// ---------------------------------------------------------------------------
template <bool FUSED>
__device__ void mma_issue_loop(const Ctx& c, const Params& p) {
  constexpr uint32_t ID_KMAJ = idesc_bf16_f32(128, 128, false, false);  // Q K^T
  constexpr uint32_t ID_BMN = idesc_bf16_f32(128, 128, false, true);    // Q~ S, P V
  constexpr uint32_t ID_AMN = idesc_bf16_f32(128, 128, true, true);     // K~^T V
  const uint32_t sbase = c.sbase;
  const uint32_t kvb = sbase + OFF_KVB;
  uint32_t q_it = 0, k_it = 0, v_it = 0, w_it = 0, gb = 0;
  uint32_t ready_n = 0, kvb_n = 0, kvfree_n = 0, p1_it = 0;

  // S/P buffer (gidx & 1) <- Q K^T for global phase-2 block gidx.
  auto issue_S = [&](uint32_t qi, uint32_t ki, uint32_t gidx) -> bool {
    const uint32_t qs = qi & 1u, ks = ki & 1u, buf = gidx & 1u;
    if (!wait_bar(c, p, B_QF + qs, (qi >> 1) & 1u)) return false;
    if (!wait_bar(c, p, B_KF + ks, (ki >> 1) & 1u)) return false;
    // fused layer: group X activates (SiLU) Q and K in place first
    if (FUSED && !wait_bar(c, p, B_ACT + buf, (gidx >> 1) & 1u)) return false;
    if (gidx >= 2 && !wait_bar(c, p, B_SE + buf, ((gidx >> 1) - 1) & 1u)) return false;
    LA_TRACE_EVENT(4, gidx);
    tc_fence_after();
    const uint32_t qa = sbase + OFF_Q + qs * TILE, ka = sbase + OFF_K + ks * TILE;
#pragma unroll
    for (uint32_t kk = 0; kk < 8; ++kk) {
      const uint32_t off = (kk >> 2) * PLANE + (kk & 3u) * 32u;
      mma_ss(c.tmem + TM_S0 + buf * 128u, sdesc_sw128(qa + off, 16, 1024),
             sdesc_sw128(ka + off, 16, 1024), ID_KMAJ, kk > 0);
    }
    mma_commit(&c.bar[B_SF + buf]);
    return true;
  };

  for (;;) {
    const uint32_t ws = w_it & 1u;
    if (!wait_bar(c, p, B_WF + ws, (w_it >> 1) & 1u)) return;
    const int w = static_cast<int>(c.misc[1 + ws]);
    mbar_arrive(&c.bar[B_WE + ws]);
    ++w_it;
    Item it;
    if (!get_item(p, c.misc, w, it)) return;
    if (!wait_bar(c, p, B_KV_FREE, kvfree_n++ & 1u)) return;
    if (it.phase1) {
      for (int b = 0; b < it.nb; ++b) {
        const uint32_t slot = p1_it % P1_SLOTS;
        if (!wait_bar(c, p, B_KT + slot, (p1_it / P1_SLOTS) & 1u)) return;
        tc_fence_after();
        const uint32_t ka = sbase + p1_base(slot), va = ka + TILE;
#pragma unroll
        for (uint32_t kk = 0; kk < 8; ++kk)
          mma_ss(c.tmem + TM_KV, sdesc_sw128(ka + kk * 2048u, PLANE, 1024),
                 sdesc_sw128(va + kk * 2048u, PLANE, 1024), ID_AMN, (b > 0) || (kk > 0));
        mma_commit(&c.bar[B_P1E + slot]);
        ++p1_it;
      }
      mma_commit(&c.bar[B_AGG_FULL]);
      LA_TRACE_EVENT(21, w_it);
    }
    const uint32_t q0 = q_it, k0 = k_it, v0 = v_it, g0 = gb;
    const uint32_t nb = it.p2 ? static_cast<uint32_t>(it.nb) : 0u;
    if (nb > 0 && !issue_S(q0, k0, g0)) return;
    for (uint32_t n = 0; n < nb; ++n) {
      const uint32_t g = g0 + n;
      const uint32_t ks = (k0 + n) & 1u, vs = (v0 + n) & 1u;
      if (!wait_bar(c, p, B_READY, ready_n++ & 1u)) return;
      LA_TRACE_EVENT(3, g);
      // (the next block's scores follow this block's products)
      if (!wait_bar(c, p, B_KVB_READY, kvb_n++ & 1u)) return;
      LA_TRACE_EVENT(5, g);
      if (!wait_bar(c, p, B_VF + vs, ((v0 + n) >> 1) & 1u)) return;
      LA_TRACE_EVENT(6, g);
      tc_fence_after();
      const uint32_t ka = sbase + OFF_K + ks * TILE;
      const uint32_t va = sbase + OFF_V + vs * TILE;
      // state += (decayed K)^T V
#pragma unroll
      for (uint32_t kk = 0; kk < 8; ++kk)
        mma_ss(c.tmem + TM_KV, sdesc_sw128(ka + kk * 2048u, PLANE, 1024),
               sdesc_sw128(va + kk * 2048u, PLANE, 1024), ID_AMN, 1);
      if (g >= 1 && !wait_bar(c, p, B_O_EMPTY, (g - 1) & 1u)) return;
      LA_TRACE_EVENT(7, g);
      tc_fence_after();
      // O = (gamma^(i+1) Q) S_bf16, the decayed Q read from TMEM
      const uint32_t abase = c.tmem + TM_S0 + (g & 1u) * 128u;
#pragma unroll
      for (uint32_t kk = 0; kk < 8; ++kk)
        mma_ts(c.tmem + TM_O, abase + 32u + (kk >> 2) * 64u + (kk & 3u) * 8u,
               sdesc_sw128(kvb + kk * 2048u, PLANE, 1024), ID_BMN, kk > 0);
      // The K tile is dead once the state update finishes.
      mma_commit(&c.bar[B_KVO_DONE]);
      mma_commit(&c.bar[B_KE + ks]);
      // O += P V, P read from TMEM (bf16 pairs: j < 64 at +0, j >= 64 at +64)
#pragma unroll
      for (uint32_t kk = 0; kk < 8; ++kk)
        mma_ts(c.tmem + TM_O, abase + (kk >> 2) * 64u + (kk & 3u) * 8u,
               sdesc_sw128(va + kk * 2048u, PLANE, 1024), ID_BMN, 1);
      mma_commit(&c.bar[B_O_FULL]);
      mma_commit(&c.bar[B_SE + (g & 1u)]);
      LA_TRACE_EVENT(8, g);
      if (n + 1 < nb && !issue_S(q0 + n + 1, k0 + n + 1, g + 1)) return;
      // The V tile is released by group Y after it has staged the output there.
    }
    q_it += nb;
    k_it += nb;
    v_it += nb;
    gb += nb;
  }
}

// Runs the issue loop, then waits (bounded) until every MMA it issued has
// completed, so TMEM is never released under a running MMA.
template <bool FUSED>
__device__ void mma_issuer(const Ctx& c, const Params& p) {
  mma_issue_loop<FUSED>(c, p);
  mma_commit(&c.bar[B_DRAIN]);
  mbar_wait(&c.bar[B_DRAIN], 0, p.wait_limit_ns);
}

// ---------------------------------------------------------------------------
// fp32 rows of 32 columns to and from global memory (states).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ld_global32(const float* src, uint32_t (&x)[32]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = __ldcg(s4 + i);
    x[4 * i] = __float_as_uint(v.x);
    x[4 * i + 1] = __float_as_uint(v.y);
    x[4 * i + 2] = __float_as_uint(v.z);
    x[4 * i + 3] = __float_as_uint(v.w);
  }
}

__device__ __forceinline__ void st_global32(float* dst, const uint32_t (&x)[32]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    __stcg(d4 + i, make_float4(__uint_as_float(x[4 * i]), __uint_as_float(x[4 * i + 1]),
                               __uint_as_float(x[4 * i + 2]), __uint_as_float(x[4 * i + 3])));
}

// Chunk states in the scan scratch use a thread-blocked layout: the float4 that
// thread (row r, half hf) holds as its i-th vector of pass h lives at float4
// index ((hf * 2 + h) * 8 + i) * 128 + r, so each warp-wide access covers 512
// contiguous bytes.
__device__ __forceinline__ void ld_scan32(const float* base, uint32_t r, uint32_t hf, uint32_t h,
                                          uint32_t (&x)[32]) {
  const float4* s4 = reinterpret_cast<const float4*>(base);
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    const float4 v = __ldcg(s4 + ((hf * 2u + h) * 8u + i) * 128u + r);
    x[4 * i] = __float_as_uint(v.x);
    x[4 * i + 1] = __float_as_uint(v.y);
    x[4 * i + 2] = __float_as_uint(v.z);
    x[4 * i + 3] = __float_as_uint(v.w);
  }
}

__device__ __forceinline__ void st_scan32(float* base, uint32_t r, uint32_t hf, uint32_t h,
                                          const uint32_t (&x)[32]) {
  float4* d4 = reinterpret_cast<float4*>(base);
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i)
    __stcg(d4 + ((hf * 2u + h) * 8u + i) * 128u + r,
           make_float4(__uint_as_float(x[4 * i]), __uint_as_float(x[4 * i + 1]),
                       __uint_as_float(x[4 * i + 2]), __uint_as_float(x[4 * i + 3])));
}

// ---------------------------------------------------------------------------
// Group X: decay-causal mask, the in-place operand decays and the split
// scan's chained entering states.
// ---------------------------------------------------------------------------
template <bool REV, bool FUSED>
__device__ void group_x(const Ctx& c, const Params& p) {
  const uint32_t t = threadIdx.x - 32u * X_WARP0;  // 0..255
  const uint32_t warp = t >> 5;
  const uint32_t r = (warp & 3u) * 32u + (t & 31u);
  const uint32_t hf = warp >> 2;
  const uint32_t lane_base = ((warp & 3u) * 32u) << 16;
  const uint32_t gtab = c.sbase + OFF_GTAB;
  uint32_t q_it = 0, k_it = 0, w_it = 0, gb = 0, xs_n = 0, p1_it = 0, chain_n = 0;
  // Split scan: an output item that starts inside its sequence enters with
  //   S(X) = gamma^(128 (X - x_lo)) S(x_lo) + sum_j gamma^(128 (X - y_j)) piece_j
  // over the published pieces that group Y's first warp has listed and seen.
  // Group X combines it (the MMA issuer waits for the state anyway): two column
  // quarters of row r per thread, half of what each of group Y's threads would
  // load, into the state's bf16 copy and the TMEM state.
  auto combine_chain = [&](const Item& it, float lam) -> bool {
    if (!cwait(c, p, B_CHAIN, chain_n++ & 1u)) return false;
    const int n = static_cast<int>(c.misc[18]);
    const int64_t span = it.t0 / BLK;  // X - x_lo, in blocks
    const float g_all = expf(-lam * static_cast<float>(span * BLK));
    const float g0 = expf(-lam * static_cast<float>(min(BLK, it.Lc)));
    const float* init = p.init_state && static_cast<int>(r) < p.D
                            ? p.init_state + static_cast<int64_t>(it.seq) * p.D * p.E +
                                  static_cast<int64_t>(r) * p.E
                            : nullptr;
    const float* prefix = cta_role(p) ? p.prefix1 : p.prefix;
    const uint32_t t_kv = c.tmem + lane_base + TM_KV;
#pragma unroll 1
    for (uint32_t qq = 0; qq < 2; ++qq) {
      const uint32_t q = 2u * hf + qq;
      uint32_t prev[32];
      if (init && 32 * static_cast<int>(q) < p.E) {
        ld_global32(init + 32 * q, prev);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) prev[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) prev[i] = __float_as_uint(g_all * __uint_as_float(prev[i]));
#pragma unroll 1
      for (int j = 0; j < n; ++j) {
        uint32_t part[32];
        ld_scan32(prefix + static_cast<int64_t>(c.chain[2 * j]) * (HD * HD), r, q >> 1, q & 1u, part);
        const float w = expf(-lam * static_cast<float>(static_cast<int>(c.chain[2 * j + 1]) * BLK));
#pragma unroll
        for (int i = 0; i < 32; ++i)
          prev[i] = __float_as_uint(fmaf(w, __uint_as_float(part[i]), __uint_as_float(prev[i])));
      }
      store_half_bf16(c.sbase + OFF_KVB + hf * PLANE + r * 128u, r, qq, prev, 1.f);
      tmem_st32_scaled(t_kv + 32u * q, prev, g0);
    }
    fence_proxy_async_smem();
    tmem_wait_st();
    tc_fence_before();
    warp_arrive(&c.bar[B_CHAIN_DONE]);
    return true;
  };
  // fused layer: SiLU on the Q and K tiles of phase-2 block gidx in place, then
  // the MMA issuer may compute their scores
  auto activate_qk = [&](uint32_t qi, uint32_t ki, uint32_t gidx) -> bool {
    if (!cwait(c, p, B_QF + (qi & 1u), (qi >> 1) & 1u) ||
        !cwait(c, p, B_KF + (ki & 1u), (ki >> 1) & 1u))
      return false;
    silu_row(c.sbase + OFF_Q + (qi & 1u) * TILE + hf * PLANE + r * 128u, r, 1.f);
    silu_row(c.sbase + OFF_K + (ki & 1u) * TILE + hf * PLANE + r * 128u, r, 1.f);
    fence_proxy_async_smem();
    warp_arrive(&c.bar[B_ACT + (gidx & 1u)]);
    return true;
  };
  for (;;) {
    const uint32_t ws = w_it & 1u;
    if (!cwait(c, p, B_WF + ws, (w_it >> 1) & 1u)) break;
    const int w = static_cast<int>(c.misc[1 + ws]);
    warp_arrive(&c.bar[B_WE + ws]);
    ++w_it;
    Item it;
    if (!get_item(p, c.misc, w, it)) break;
    const float lam = p.slopes[it.seq % p.H];

    // decay table: gtab[u] = gamma^(127-u) for u <= 127, 0 above (the causal mask)
    if (!gsync(c, p, B_XSYNC, xs_n)) break;  // the previous item's table is no longer read
    sts32f(gtab + 4u * t, t <= 127u ? expf(-lam * static_cast<float>(127u - t)) : 0.f);
    if (!gsync(c, p, B_XSYNC, xs_n)) break;

    bool ok = true;
    if (it.enter && p.mode == MODE_SPLIT_SCAN) ok = combine_chain(it, lam);
    if (it.phase1 && ok) {  // K rows decayed to the chunk end: gamma^(Lc-1-j)
      for (int b = 0; b < it.nb && ok; ++b) {
        const uint32_t slot = p1_it % P1_SLOTS;
        if (!cwait(c, p, B_P1F + slot, (p1_it / P1_SLOTS) & 1u)) { ok = false; break; }
        // reversed chunk-local index of this tile row (REV: row r is 127 - r)
        const int jc = b * BLK + static_cast<int>(REV ? 127u - r : r);
        const float f = jc < it.Lc ? expf(-lam * static_cast<float>(it.Lc - 1 - jc)) : 0.f;
        if (FUSED) {  // SiLU on k (with its decay) and on v
          silu_row(c.sbase + p1_base(slot) + hf * PLANE + r * 128u, r, f);
          silu_row(c.sbase + p1_base(slot) + TILE + hf * PLANE + r * 128u, r, 1.f);
        } else {
          scale_row(c.sbase + p1_base(slot) + hf * PLANE + r * 128u, r, f);
        }
        fence_proxy_async_smem();
        warp_arrive(&c.bar[B_KT + slot]);
        if (t == 0) LA_TRACE_EVENT(22, p1_it);
        ++p1_it;
      }
    }
    if (FUSED && it.p2 && it.nb > 0 && ok) ok = activate_qk(q_it, k_it, gb);
    for (int n = 0; n < (it.p2 ? it.nb : 0) && ok; ++n) {
      const uint32_t g = gb;
      const int len = min(BLK, it.Lc - n * BLK);
      const uint32_t qs = q_it & 1u, ks = k_it & 1u;
      if (!cwait(c, p, B_SF + (g & 1u), (g >> 1) & 1u) ||
          !cwait(c, p, B_QF + qs, (q_it >> 1) & 1u) ||
          !cwait(c, p, B_KF + ks, (k_it >> 1) & 1u)) { ok = false; break; }
      if (t == 0) LA_TRACE_EVENT(9, g);
      tc_fence_after();
      const uint32_t t_s = c.tmem + lane_base + TM_S0 + (g & 1u) * 128u + hf * 64u;
      // P_ij = S_ij * gtab[j - r + 127] (zero above the diagonal); rows past len
      // have zero scores (zero-filled Q), so they give zero P as well.  In the
      // quarter with every column above every row (hf = 1, rows < 64) P is 0.
      uint32_t pk[32];
      // causal: P_rc = S_rc gamma^(r-c) for c <= r; anti-causal (rows in
      // reversed order): P_rc = S_rc gamma^(c-r) for c >= r.  The quadrant
      // where the condition fails for every (r, c) is zero.
      if (REV ? (hf == 0 && (warp & 3u) >= 2) : (hf == 1 && (warp & 3u) < 2)) {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      } else {
#pragma unroll
        for (uint32_t half = 0; half < 2; ++half) {
          uint32_t sc[32];
          tmem_ld32(t_s + half * 32u, sc);
          tmem_wait_ld();
          if (REV) {
            const uint32_t u0 = gtab + 4u * (r + 127u - hf * 64u - half * 32u);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[16 * half + i] =
                  pack_bf16x2(__uint_as_float(sc[2 * i]) * lds32f(u0 - 8u * i),
                              __uint_as_float(sc[2 * i + 1]) * lds32f(u0 - 8u * i - 4u));
          } else {
            const uint32_t u0 = gtab + 4u * (hf * 64u + half * 32u + 127u - r);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[16 * half + i] =
                  pack_bf16x2(__uint_as_float(sc[2 * i]) * lds32f(u0 + 8u * i),
                              __uint_as_float(sc[2 * i + 1]) * lds32f(u0 + 8u * i + 4u));
          }
        }
      }
      tmem_st32(t_s, pk);
      if (FUSED) {  // SiLU on V in place before the state and PV products read it
        if (!cwait(c, p, B_VF + qs, (q_it >> 1) & 1u)) { ok = false; break; }
        silu_row(c.sbase + OFF_V + qs * TILE + hf * PLANE + r * 128u, r, 1.f);
      }
      // gamma^(r+1) Q (bf16) into the S buffer's free columns; the Q tile is then dead
      {
        // gamma^(i+1) for the (reversed, if REV) local index i of row r
        const float fq = lds32f(gtab + 4u * (REV ? r : 127u - r)) * lds32f(gtab + 4u * 126u);
        const uint32_t qrow = c.sbase + OFF_Q + qs * TILE + hf * PLANE + r * 128u;
        uint32_t qv[32];
#pragma unroll
        for (uint32_t ch = 0; ch < 8; ++ch) {
          const uint4 x = lds128(qrow + ((ch ^ (r & 7u)) << 4));
          qv[4 * ch + 0] = scale_bf16x2(x.x, fq);
          qv[4 * ch + 1] = scale_bf16x2(x.y, fq);
          qv[4 * ch + 2] = scale_bf16x2(x.z, fq);
          qv[4 * ch + 3] = scale_bf16x2(x.w, fq);
        }
        tmem_st32(t_s + 32u, qv);
        // The Q tile is dead now.  Its release comes after the TMEM store
        // (which consumes every load above, so they have completed) and a
        // proxy fence (these generic-proxy reads are ordered before the TMA
        // write of a later tile into the slot, an async-proxy access): when the
        // release came straight after the loads, the producer's next Q tile
        // could land while a warp's reads were still in flight, and the inter
        // term of that warp's rows then used rows of the wrong tile.
        fence_proxy_async_smem();
        warp_arrive(&c.bar[B_QE + qs]);
      }
      // gamma^(len-1-r) K (0 past len) in place
      // gamma^(len-1-j) for the local index j of row r (0 past len)
      const float fk = lds32f(gtab + 4u * (REV ? 255u - static_cast<uint32_t>(len) - r
                                               : 128u - static_cast<uint32_t>(len) + r));
      scale_row(c.sbase + OFF_K + ks * TILE + hf * PLANE + r * 128u, r, fk);
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(&c.bar[B_READY]);
      if (t == 0) LA_TRACE_EVENT(10, g);
      ++q_it;
      ++k_it;
      ++gb;
      if (FUSED && n + 1 < it.nb && !activate_qk(q_it, k_it, gb)) { ok = false; break; }
    }
    if (!ok) break;
  }
}

// ---------------------------------------------------------------------------
// Group Y: entering states, state copy/decay, chunk scan, epilogue.
// ---------------------------------------------------------------------------
template <int RANK, bool REV, bool FUSED>
__device__ void group_y(const Ctx& c, const Params& p, const CUtensorMap* to) {
  const uint32_t t = threadIdx.x - 32u * Y_WARP0;  // 0..127
  const uint32_t r = t;                            // TMEM lane / tile row
  const uint32_t lane_base = ((t >> 5) * 32u) << 16;
  const uint32_t t_kv = c.tmem + lane_base + TM_KV;
  const uint32_t t_o = c.tmem + lane_base + TM_O;
  // the caller's states are [seq][D][E]; rows r >= D of the 128 x 128 TMEM
  // state are zero (zero-filled K columns) and never read or written
  const int64_t row_off = static_cast<int64_t>(r) * p.E;
  const bool row_in = static_cast<int>(r) < p.D;
  const int64_t state_elems = static_cast<int64_t>(p.D) * p.E;
  const bool leader = (t == 0);
  const uint64_t pol_out = policy_evict_first();
  uint32_t v_it = 0, w_it = 0, gb = 0, agg_n = 0, ys_n = 0, chain_done_n = 0;
  // this CTA's scratch and plain-store output (the second role's in a paired launch)
  const bool role1 = cta_role(p) != 0;
  float* const prefix = role1 ? p.prefix1 : p.prefix;
  unsigned long long* const flags = role1 ? p.flags1 : p.flags;
  float* const out = role1 ? p.out1 : p.out;
  // kvb row address of column quarter q (32 columns): plane q / 2, chunks 4 (q % 2)..
  auto kvb_row = [&](uint32_t q) { return c.sbase + OFF_KVB + (q >> 1) * PLANE + r * 128u; };

  for (;;) {
    const uint32_t ws = w_it & 1u;
    if (!cwait(c, p, B_WF + ws, (w_it >> 1) & 1u)) break;
    const int w = static_cast<int>(c.misc[1 + ws]);
    warp_arrive(&c.bar[B_WE + ws]);
    ++w_it;
    Item it;
    if (!get_item(p, c.misc, w, it)) break;
    const float lam = p.slopes[it.seq % p.H];
    tc_fence_before();
    warp_arrive(&c.bar[B_KV_FREE]);  // done with the previous item's state
    if (leader) LA_TRACE_EVENT(15, w_it);

    // ---- entering state; publication of this chunk's inclusive state ----
    const float* scan_src = nullptr;  // previous chunk's state (scan layout)
    const float* init_src = nullptr;  // caller's initial state (row layout)
    // split scan: the entering state chains the published local states of the
    // stream pieces [s F, X) (X = stream position of this item's first block)
    const bool chain = it.enter && p.mode == MODE_SPLIT_SCAN;
    const int64_t G = vgrid(p);
    const int64_t x_lo = static_cast<int64_t>(it.seq) * p.F;
    const int64_t x_hi = x_lo + it.t0 / BLK;
    if (it.enter) {
      if (t < 32) {  // the group's first warp waits
        // The chain's pieces follow from the plan alone: lane 0 lists them
        // (slot, distance to X), then every lane waits for one piece's flag,
        // so the pieces' publication latencies overlap instead of adding up.
        if (chain && t == 0) {
          uint32_t m = 0;
          for (int64_t x = x_lo; x < x_hi;) {
            if (m == CHAIN_MAX) {  // excluded by the host's plan; no wrong result
              fail(c, p, 4);
              m = 0;
              break;
            }
            const int64_t y = s1_next(p, G, x);
            c.chain[2 * m] = static_cast<uint32_t>(s1_slot(p, G, x));
            c.chain[2 * m + 1] = static_cast<uint32_t>(x_hi - y);
            ++m;
            x = y;
          }
          c.misc[18] = m;
        }
        __syncwarp();
        const uint32_t n = chain ? c.misc[18] : 1u;
        const unsigned long long* f =
            t < n ? flags + (chain ? static_cast<int>(c.chain[2 * t]) : it.enter_slot) : nullptr;
        bool seen = f == nullptr;
        const uint64_t t0 = globaltimer_ns();
        uint32_t spins = 0;
        for (;;) {
          if (!seen) seen = ld_acquire_gpu(f) == it.enter_val;
          if (__all_sync(0xffffffffu, seen)) break;
          // spins is the same in every lane, so the lanes decide together
          if ((++spins & 15u) == 0 &&
              __any_sync(0xffffffffu, aborted(c) || globaltimer_ns() - t0 > p.wait_limit_ns)) {
            if (t == 0) fail(c, p, 2);
            break;
          }
        }
        // group X combines a chain (it waits for the list and the flags): the
        // warp barrier orders every lane's acquire before lane 0's release
        __syncwarp();
        if (chain && t == 0) mbar_arrive(&c.bar[B_CHAIN]);
      }
      if (!gsync(c, p, B_YSYNC, ys_n)) break;
      if (!chain) scan_src = prefix + static_cast<int64_t>(it.enter_slot) * (HD * HD);
    }
    // the caller's initial state enters at block 0 of a sequence (or through
    // the chain); never into a local state -- except in the state pass, where
    // the first chunk's inclusive state starts from it
    if (p.init_state && (it.p2 || p.state_only) && !it.enter && row_in)
      init_src = p.init_state + static_cast<int64_t>(it.seq) * state_elems + row_off;
    if (leader) LA_TRACE_EVENT(16, w_it);
    if (it.phase1 && !cwait(c, p, B_AGG_FULL, agg_n++ & 1u)) break;
    if (leader) LA_TRACE_EVENT(17, w_it);
    if (chain) {  // group X has combined the entering state into KVB and TMEM
      if (!cwait(c, p, B_CHAIN_DONE, chain_done_n++ & 1u)) break;
      tc_fence_after();
    } else {
      tc_fence_after();
      const float gL = expf(-lam * static_cast<float>(it.Lc));
      const float g0 = expf(-lam * static_cast<float>(min(BLK, it.Lc)));
      float* pub = prefix + static_cast<int64_t>(it.pub_slot) * (HD * HD);
#pragma unroll 1
      for (uint32_t q = 0; q < 4; ++q) {
        uint32_t prev[32];
        if (scan_src) {
          ld_scan32(scan_src, r, q >> 1, q & 1u, prev);
        } else if (init_src && 32 * static_cast<int>(q) < p.E) {
          ld_global32(init_src + 32 * q, prev);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) prev[i] = 0u;
        }
        if (it.phase1) {
          uint32_t agg[32];
          tmem_ld32(t_kv + 32u * q, agg);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            agg[i] = __float_as_uint(fmaf(gL, __uint_as_float(prev[i]), __uint_as_float(agg[i])));
          if (p.state_only && it.last) {  // the state after the sequence, to the caller
            if (row_in && 32 * static_cast<int>(q) < p.E)
              st_global32(p.final_state + static_cast<int64_t>(it.seq) * state_elems + row_off +
                              32 * q,
                          agg);
          } else {
            st_scan32(pub, r, q >> 1, q & 1u, agg);
          }
        }
        if (it.p2) {
          store_half_bf16(kvb_row(q), r, q & 1u, prev, 1.f);
          tmem_st32_scaled(t_kv + 32u * q, prev, g0);
        }
      }
    }
    if (leader) LA_TRACE_EVENT(18, w_it);
    if (it.phase1 && !(p.state_only && it.last)) {  // (the state pass's last chunk has no successor)
      // the group's stores are ordered before the leader's fence and release
      if (!gsync(c, p, B_YSYNC, ys_n)) break;
      if (leader) {
        __threadfence();
        st_release_gpu(flags + it.pub_slot, it.pub_val);
      }
    }
    if (leader) LA_TRACE_EVENT(19, w_it);
    if (!it.p2) continue;  // a local-state item has no outputs
    fence_proxy_async_smem();
    tmem_wait_st();
    tc_fence_before();
    warp_arrive(&c.bar[B_KVB_READY]);
    if (leader) LA_TRACE_EVENT(20, w_it);

    // where the state after the item's last block goes: the caller's final
    // state (row layout) or a balanced split's hand-over slot (scan layout)
    float* const fin_dst = it.last && p.final_state && row_in
                               ? p.final_state + static_cast<int64_t>(it.seq) * state_elems + row_off
                               : nullptr;
    float* const pub_dst = it.publish ? prefix + static_cast<int64_t>(it.pub_slot) * (HD * HD) : nullptr;
    unsigned long long* const pub_flag = it.publish ? flags + it.pub_slot : nullptr;
    const unsigned long long pub_val = it.pub_val;
    bool ok = true;
    for (int n = 0; n < it.nb && ok; ++n) {
      const uint32_t g = gb;
      const uint32_t vs = v_it & 1u;
      // (B) state: bf16 copy for the next block's inter term, decay in TMEM
      if (!cwait(c, p, B_KVO_DONE, g & 1u)) { ok = false; break; }
      if (leader) LA_TRACE_EVENT(11, g);
      tc_fence_after();
      {
        const bool more = n + 1 < it.nb;
        const float gnext =
            more ? expf(-lam * static_cast<float>(min(BLK, it.Lc - (n + 1) * BLK))) : 1.f;
        const bool fin = !more && fin_dst != nullptr;
        const bool pub = !more && pub_dst != nullptr;
#pragma unroll 1
        for (uint32_t q = 0; q < 4; ++q) {
          uint32_t kv[32];
          tmem_ld32(t_kv + 32u * q, kv);
          tmem_wait_ld();
          if (more) {
            store_half_bf16(kvb_row(q), r, q & 1u, kv, 1.f);
            tmem_st32_scaled(t_kv + 32u * q, kv, gnext);
          } else if (fin) {
            if (32 * static_cast<int>(q) < p.E) st_global32(fin_dst + 32 * q, kv);
          } else if (pub) {
            st_scan32(pub_dst, r, q >> 1, q & 1u, kv);
          }
        }
        if (more) {
          fence_proxy_async_smem();
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(&c.bar[B_KVB_READY]);
        } else if (pub) {
          // the state goes to the CTA that continues this sequence: the
          // group's stores are ordered before the leader's fence and release
          if (!gsync(c, p, B_YSYNC, ys_n)) { ok = false; break; }
          if (leader) {
            __threadfence();
            st_release_gpu(pub_flag, pub_val);
          }
        }
        if (leader) LA_TRACE_EVENT(12, g);
      }
      // (C) epilogue: O -> swizzled staging in this block's V slot (dead once O
      //     is complete), 64 columns at a time -> TMA store.
      if (!cwait(c, p, B_O_FULL, g & 1u)) { ok = false; break; }
      if (leader) LA_TRACE_EVENT(13, g);
      tc_fence_after();
      const uint32_t vtile = c.sbase + OFF_V + vs * TILE;
      const uint8_t* vtile_g = c.sm + OFF_V + vs * TILE;
      const int row = tile_row(p, it.t0 + n * BLK, REV);
      if (REV && row < 0) {
        // The block holding token 0 of an anti-causal run starts at a
        // negative row, where a TMA store may not start: plain stores of the
        // rows that exist, straight from TMEM.  The V slot is not needed.
        const int tok = row + static_cast<int>(r);
        float* dst = tok >= 0 ? out + (it.seq / p.H) * p.ostride[0] + (it.seq % p.H) * p.ostride[1] +
                                     static_cast<int64_t>(tok) * p.ostride[2]
                              : nullptr;
#pragma unroll 1
        for (uint32_t qq = 0; qq < 4; ++qq) {
          uint32_t o[32];
          tmem_ld32(t_o + 32u * qq, o);
          tmem_wait_ld();
          if (dst && 32 * static_cast<int>(qq) < p.E) st_global32(dst + 32 * qq, o);
        }
        tc_fence_before();
        warp_arrive(&c.bar[B_O_EMPTY]);
        if (leader) mbar_arrive(&c.bar[B_VE + vs]);
        if (leader) LA_TRACE_EVENT(14, g);
        ++v_it;
        ++gb;
        continue;
      }
      if (FUSED) {
        // Fused layer: y = w * o / sqrt(mean_e(o^2) + eps) * sigmoid(gate) in
        // bf16, staged in this block's V slot (128 rows x 128 bf16 = one tile,
        // laid out like the input tiles) and written by one pair of TMA stores.
        // The row's gate is first copied (cp.async) into exactly the positions
        // its outputs will take, while the row's mean square is computed; each
        // output chunk then overwrites its own gate chunk.
        const int tok = row + static_cast<int>(r);
        const uint16_t* grow = tok < p.N ? p.gate + (it.seq / p.H) * p.gstride[0] +
                                               (it.seq % p.H) * p.gstride[1] +
                                               static_cast<int64_t>(tok) * p.gstride[2]
                                         : nullptr;
        const uint32_t srow = vtile + r * 128u;
        if (grow) {
#pragma unroll
          for (uint32_t ch = 0; ch < 16; ++ch)  // 16-byte chunk ch: plane ch / 8, chunk ch % 8
            if (static_cast<int>(8 * ch) < p.E)
              cp_async16(srow + (ch >> 3) * PLANE + (((ch & 7u) ^ (r & 7u)) << 4), grow + 8 * ch);
        }
        float ss = 0.f;
#pragma unroll 1
        for (uint32_t qq = 0; qq < 4; ++qq) {
          uint32_t o[32];
          tmem_ld32(t_o + 32u * qq, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            ss = fmaf(__uint_as_float(o[i]), __uint_as_float(o[i]), ss);
        }
        const float rinv = rsqrtf(ss / static_cast<float>(p.E) + p.eps);
        const float* wrow = p.norm_w + static_cast<int64_t>(it.seq % p.H) * p.E;
        if (leader) LA_TRACE_EVENT(23, g);
        cp_async_wait_all();
        if (leader) LA_TRACE_EVENT(24, g);
#pragma unroll 1
        for (uint32_t qq = 0; qq < 4; ++qq) {
          uint32_t o[32];
          tmem_ld32(t_o + 32u * qq, o);
          tmem_wait_ld();
          if (qq == 3) {  // every TMEM read of O done
            tc_fence_before();
            warp_arrive(&c.bar[B_O_EMPTY]);
          }
#pragma unroll
          for (uint32_t cc = 0; cc < 4; ++cc) {  // 8 columns at a time
            const int col = 32 * static_cast<int>(qq) + 8 * static_cast<int>(cc);
            const uint32_t lc = (qq & 1u) * 4u + cc;  // 16-byte chunk within the 64-column plane
            const uint32_t addr = srow + (qq >> 1) * PLANE + ((lc ^ (r & 7u)) << 4);
            float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
            uint4 gv = make_uint4(0u, 0u, 0u, 0u);
            if (col < p.E) {
              w0 = __ldg(reinterpret_cast<const float4*>(wrow + col));
              w1 = __ldg(reinterpret_cast<const float4*>(wrow + col + 4));
              if (grow) gv = lds128(addr);
            }
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t yw[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float a = wv[2 * j] * rinv * __uint_as_float(o[8 * cc + 2 * j]) *
                              sigmoid_hw(bf16lo_to_f32(gw[j]));
              const float b = wv[2 * j + 1] * rinv * __uint_as_float(o[8 * cc + 2 * j + 1]) *
                              sigmoid_hw(bf16hi_to_f32(gw[j]));
              yw[j] = pack_bf16x2(a, b);
            }
            sts128(addr, make_uint4(yw[0], yw[1], yw[2], yw[3]));
          }
        }
        fence_proxy_async_smem();
        if (leader) LA_TRACE_EVENT(25, g);
        if (!gsync(c, p, B_YSYNC, ys_n)) { ok = false; break; }
        if (leader) {
          tile_store<RANK>(to, vtile_g, 0, row, it.seq, it.seq % p.H, it.seq / p.H, p.cslot[3],
                           pol_out);
          tile_store<RANK>(to, vtile_g + PLANE, 64, row, it.seq, it.seq % p.H, it.seq / p.H,
                           p.cslot[3], pol_out);
          bulk_commit_group();
          LA_TRACE_EVENT(26, g);
          bulk_wait_group_read<0>();
          mbar_arrive(&c.bar[B_VE + vs]);
        }
        if (leader) LA_TRACE_EVENT(14, g);
        ++v_it;
        ++gb;
        continue;
      }
      uint32_t o0[32], o1[32];
      tmem_ld32(t_o, o0);
      tmem_ld32(t_o + 32u, o1);
      tmem_wait_ld();
      store_row_f32(vtile + r * 128u, r, o0);
      store_row_f32(vtile + PLANE + r * 128u, r, o1);
      fence_proxy_async_smem();
      if (!gsync(c, p, B_YSYNC, ys_n)) { ok = false; break; }
      if (leader) {
        tile_store<RANK>(to, vtile_g, 0, row, it.seq, it.seq % p.H, it.seq / p.H, p.cslot[3],
                         pol_out);
        tile_store<RANK>(to, vtile_g + PLANE, 32, row, it.seq, it.seq % p.H, it.seq / p.H,
                         p.cslot[3], pol_out);
        bulk_commit_group();
        LA_TRACE_EVENT(23, g);
      }
      tmem_ld32(t_o + 64u, o0);
      tmem_ld32(t_o + 96u, o1);
      tmem_wait_ld();
      tc_fence_before();
      warp_arrive(&c.bar[B_O_EMPTY]);
      if (leader) LA_TRACE_EVENT(24, g);
      if (leader) bulk_wait_group_read<0>();
      if (leader) LA_TRACE_EVENT(25, g);
      if (!gsync(c, p, B_YSYNC, ys_n)) { ok = false; break; }
      store_row_f32(vtile + r * 128u, r, o0);
      store_row_f32(vtile + PLANE + r * 128u, r, o1);
      fence_proxy_async_smem();
      if (!gsync(c, p, B_YSYNC, ys_n)) { ok = false; break; }
      if (leader) {
        tile_store<RANK>(to, vtile_g, 64, row, it.seq, it.seq % p.H, it.seq / p.H, p.cslot[3],
                         pol_out);
        tile_store<RANK>(to, vtile_g + PLANE, 96, row, it.seq, it.seq % p.H, it.seq / p.H,
                         p.cslot[3], pol_out);
        bulk_commit_group();
        LA_TRACE_EVENT(26, g);
        bulk_wait_group_read<0>();
        mbar_arrive(&c.bar[B_VE + vs]);
      }
      if (leader) LA_TRACE_EVENT(14, g);
      ++v_it;
      ++gb;
    }
    if (!ok) break;
  }
  if (leader) bulk_wait_group<0>();
}

// 14 warps on 4 SM sub-partitions (16K registers each, at most 4 warps on one)
// leave up to 128 registers per thread.
// RANK: 3 for contiguous head-major q, k, v, out; 4 for strided layouts.
// REV: anti-causal (o_t sums s >= t), the same blocked form in reversed time.
// FUSED: the layer around the operator (SiLU on q, k, v in shared memory;
// per-head RMSNorm, weight and sigmoid gate on the output, stored as bf16).
template <int RANK, bool REV, bool FUSED>
__global__ void __launch_bounds__(THREADS, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                    const __grid_constant__ CUtensorMap tq1, const __grid_constant__ CUtensorMap tk1,
                    const __grid_constant__ CUtensorMap tv1, const __grid_constant__ CUtensorMap to1,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Ctx c;
  c.sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
  c.sbase = smem_u32(c.sm);
  c.bar = reinterpret_cast<uint64_t*>(c.sm + OFF_BAR);
  c.misc = reinterpret_cast<volatile uint32_t*>(c.sm + OFF_MISC);
  c.chain = reinterpret_cast<volatile uint32_t*>(c.sm + OFF_CHAIN);
  const uint32_t warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.bar[B_QF + i], 1);
      mbar_init(&c.bar[B_QE + i], X_WARPS);
      mbar_init(&c.bar[B_KF + i], 1);
      mbar_init(&c.bar[B_KE + i], 1);
      mbar_init(&c.bar[B_VF + i], 1);
      mbar_init(&c.bar[B_VE + i], 1);
      mbar_init(&c.bar[B_SF + i], 1);
      mbar_init(&c.bar[B_SE + i], 1);
      mbar_init(&c.bar[B_ACT + i], X_WARPS);
      mbar_init(&c.bar[B_WF + i], 1);
      mbar_init(&c.bar[B_WE + i], 1 + X_WARPS + Y_WARPS);
    }
    for (int i = 0; i < P1_SLOTS; ++i) {
      mbar_init(&c.bar[B_P1F + i], 1);
      mbar_init(&c.bar[B_P1E + i], 1);
      mbar_init(&c.bar[B_KT + i], X_WARPS);
    }
    mbar_init(&c.bar[B_READY], X_WARPS);
    mbar_init(&c.bar[B_CHAIN], 1);
    mbar_init(&c.bar[B_CHAIN_DONE], X_WARPS);
    mbar_init(&c.bar[B_KVB_READY], Y_WARPS);
    mbar_init(&c.bar[B_KVO_DONE], 1);
    mbar_init(&c.bar[B_O_FULL], 1);
    mbar_init(&c.bar[B_O_EMPTY], Y_WARPS);
    mbar_init(&c.bar[B_AGG_FULL], 1);
    mbar_init(&c.bar[B_KV_FREE], Y_WARPS);
    mbar_init(&c.bar[B_XSYNC], X_WARPS);
    mbar_init(&c.bar[B_YSYNC], Y_WARPS);
    mbar_init(&c.bar[B_DRAIN], 1);
    c.misc[3] = 0;
    if (!setup_split(p, vgrid(p), vcta(p), c.misc)) {
      c.misc[4] = 0;  // cannot happen (see split_scan_setup); no work rather than wrong work
      atomicOr(p.status, 4);
    }
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(const_cast<uint32_t*>(&c.misc[0]), 512);
    tmem_relinquish();
  }
  const bool role1 = cta_role(p) != 0;
  const CUtensorMap* const mq = role1 ? &tq1 : &tq;
  const CUtensorMap* const mk = role1 ? &tk1 : &tk;
  const CUtensorMap* const mv = role1 ? &tv1 : &tv;
  const CUtensorMap* const mo = role1 ? &to1 : &to;
  if (warp == PRODUCER_WARP && lane_id() == 0) {
    prefetch_tmap(mq);
    prefetch_tmap(mk);
    prefetch_tmap(mv);
    prefetch_tmap(mo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = c.misc[0];

  if (warp == PRODUCER_WARP) {
    if (lane_id() == 0) producer<RANK, REV>(c, p, mq, mk, mv);
  } else if (warp == MMA_WARP) {
    if (lane_id() == 0) mma_issuer<FUSED>(c, p);
    __syncwarp();
  } else if (warp < Y_WARP0) {
    group_x<REV, FUSED>(c, p);
  } else {
    group_y<RANK, REV, FUSED>(c, p, mo);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(c.tmem, 512);
  }
}

}  // namespace fwd
}  // namespace la
