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
// Sequence split (chunked scan).  To give all SMs work when B*H is small, a
// sequence is cut into chunks of L tokens (L a multiple of 128).  Work item
// w = chunk * (B*H) + seq.  A chunk with a successor first computes its local
// state A_c = sum_j gamma^(Lc-1-j) k_j^T v_j over its tokens (phase 1, K/V
// kept in L2 with an evict-last hint), then takes the inclusive state of the
// previous chunk from global memory (spin on a flag, bounded in time),
// publishes its own inclusive state gamma^Lc S_prev + A_c, and finally runs
// the blocked form from S_prev (phase 2, re-reading K/V from L2).  Items are
// handed out through an atomic ticket, so every chunk's predecessor is held by
// a CTA that is already running: no co-residency assumption.
//
// Roles (320 threads, one CTA per SM):
//   warp 8      TMA producer: Q/K/V tiles into three 2-slot rings.
//   warp 9      TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 0..7  compute: mask/scale (P, gamma^(i+1) Q, decayed K), the state
//               copy to bf16 and its decay, the chunk scan, and the epilogue
//               (TMEM -> swizzled shared memory -> TMA store of fp32 out).
// TMEM (512 columns): S/P double buffer [0,256), O [256,384), state [384,512).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace la {
namespace fwd {

constexpr int BLK = 128;   // tokens per block (= MMA M)
constexpr int HD = 128;    // D = E = 128
constexpr int C_WARPS = 8;
constexpr int C_THREADS = 32 * C_WARPS;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int THREADS = 320;

constexpr uint32_t PLANE = 16384;             // 128 rows x 128 B
constexpr uint32_t TILE = 2 * PLANE;          // 128 x 128 bf16
constexpr uint32_t OFF_Q = 0;                 // 2 slots
constexpr uint32_t OFF_K = 2 * TILE;          // 2 slots
constexpr uint32_t OFF_V = 4 * TILE;          // 2 slots
constexpr uint32_t OFF_KVB = 6 * TILE;        // bf16 copy of the state (MMA B operand)
constexpr uint32_t OFF_BAR = 7 * TILE;
constexpr uint32_t OFF_GPOW = OFF_BAR + 512;  // gamma^m, m = 0..128
constexpr uint32_t OFF_MISC = OFF_GPOW + 544;
constexpr uint32_t SMEM_USED = OFF_MISC + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

constexpr uint32_t TM_S0 = 0, TM_O = 256, TM_KV = 384;

enum BarId : int {
  B_QF = 0, B_QE = 2, B_KF = 4, B_KE = 6, B_VF = 8, B_VE = 10,
  B_SF = 12, B_SE = 14,
  B_READY = 16, B_KVB_READY, B_KVO_DONE, B_O_FULL, B_O_EMPTY, B_AGG_FULL, B_KV_FREE,
  B_WF = 24, B_WE = 26,
  B_CSYNC = 28, B_DRAIN = 29,
  B_KT = 30,  // phase 1: decayed K tile ready, one per K slot (2)
  B_COUNT = 32
};

struct Params {
  const float* slopes;        // [H]
  float* prefix;              // [nseq][2][HD*HD] inclusive chunk states (chunked runs)
  int* flags;                 // [nseq][2] publication flags (chunked runs), zeroed
  int* ticket;                // work counter (chunked runs), zeroed
  const float* init_state;    // nullable [nseq][HD*HD]
  float* final_state;         // nullable [nseq][HD*HD]
  int* status;                // sticky error word
  int H, N, nseq, L, nchunks, total;
  unsigned long long wait_limit_ns;
};

struct Item {
  int seq, chunk, t0, Lc, nb;
  bool phase1;
};

__device__ __forceinline__ Item decode_item(const Params& p, int w) {
  Item it;
  it.chunk = w / p.nseq;
  it.seq = w - it.chunk * p.nseq;
  it.t0 = it.chunk * p.L;
  it.Lc = min(p.L, p.N - it.t0);
  it.nb = (it.Lc + BLK - 1) / BLK;
  it.phase1 = it.chunk + 1 < p.nchunks;
  return it;
}

__device__ __forceinline__ void st_release_gpu(int* ptr, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* ptr) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

// Multiplies the 64 bf16 of one 128-byte swizzled row by f, in place.  The
// physical chunk order (c ^ row) keeps 8 consecutive rows on distinct banks.
__device__ __forceinline__ void scale_row(uint8_t* rowp, uint32_t row, float f) {
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) {
    uint4* p = reinterpret_cast<uint4*>(rowp + ((c ^ (row & 7u)) << 4));
    uint4 x = *p;
    x.x = pack_bf16x2(bf16lo_to_f32(x.x) * f, bf16hi_to_f32(x.x) * f);
    x.y = pack_bf16x2(bf16lo_to_f32(x.y) * f, bf16hi_to_f32(x.y) * f);
    x.z = pack_bf16x2(bf16lo_to_f32(x.z) * f, bf16hi_to_f32(x.z) * f);
    x.w = pack_bf16x2(bf16lo_to_f32(x.w) * f, bf16hi_to_f32(x.w) * f);
    *p = x;
  }
}

// Writes 64 floats as bf16 into one 128-byte swizzled row (logical chunk c
// holds elements 8c..8c+7).
__device__ __forceinline__ void store_row_bf16(uint8_t* rowp, uint32_t row, const float* x) {
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) {
    uint4 u;
    u.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
    u.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
    u.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
    u.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
    *reinterpret_cast<uint4*>(rowp + ((c ^ (row & 7u)) << 4)) = u;
  }
}

// Writes 32 floats into one 128-byte swizzled fp32 row (logical chunk c holds
// elements 4c..4c+3).
__device__ __forceinline__ void store_row_f32(uint8_t* rowp, uint32_t row, const float* x) {
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c)
    *reinterpret_cast<float4*>(rowp + ((c ^ (row & 7u)) << 4)) =
        make_float4(x[4 * c + 0], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* x) {
  uint32_t a[32], b[32];
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[i] = __uint_as_float(a[i]);
    x[32 + i] = __uint_as_float(b[i]);
  }
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const float* x, float f) {
  uint32_t a[32], b[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    a[i] = __float_as_uint(x[i] * f);
    b[i] = __float_as_uint(x[32 + i] * f);
  }
  tmem_st32(taddr, a);
  tmem_st32(taddr + 32, b);
}

struct Ctx {
  uint8_t* sm;
  uint64_t* bar;
  float* gpow;
  volatile uint32_t* misc;  // [0] TMEM base, [1..2] work slots, [3] abort
  uint32_t tmem;
};

__device__ __forceinline__ bool aborted(const Ctx& c) { return c.misc[3] != 0; }

__device__ __noinline__ void fail(const Ctx& c, const Params& p, int code) {
  c.misc[3] = 1;
  atomicOr(p.status, code);
}

// Bounded wait; on time-out records the failure and returns false.
__device__ __forceinline__ bool wait_bar(const Ctx& c, const Params& p, int id, uint32_t parity) {
  if (aborted(c)) return false;
  if (mbar_wait(&c.bar[id], parity, p.wait_limit_ns)) return true;
  fail(c, p, 1);
  return false;
}

// Warp-uniform bounded wait for the compute warps: all 32 lanes take the same
// branch, so warp-collective tcgen05.ld/st that follow are never split.
__device__ __forceinline__ bool cwait(const Ctx& c, const Params& p, int id, uint32_t parity) {
  bool ok = !aborted(c) && mbar_wait(&c.bar[id], parity, p.wait_limit_ns);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && lane_id() == 0) fail(c, p, 1);
  return ok;
}

// Synchronisation of the 256 compute threads through an mbarrier (bounded,
// unlike bar.sync, so a failed wait elsewhere cannot hang the others).
__device__ __forceinline__ bool csync(const Ctx& c, const Params& p, uint32_t& n) {
  mbar_arrive(&c.bar[B_CSYNC]);
  return cwait(c, p, B_CSYNC, n++ & 1u);
}

// Next work item: dynamic ticket for chunked runs, static stride otherwise.
__device__ __forceinline__ int next_work(const Params& p, int& static_next) {
  if (p.nchunks > 1) return atomicAdd(p.ticket, 1);
  const int w = static_next;
  static_next += gridDim.x;
  return w;
}

// ---------------------------------------------------------------------------
// Producer: one thread issues every TMA load.
// ---------------------------------------------------------------------------
__device__ void producer(const Ctx& c, const Params& p, const CUtensorMap* tq,
                         const CUtensorMap* tk, const CUtensorMap* tv) {
  const uint64_t pol_first = policy_evict_first();
  const uint64_t pol_last = policy_evict_last();
  uint32_t q_it = 0, k_it = 0, v_it = 0, w_it = 0;
  int static_next = blockIdx.x;
  auto load = [&](int ring_f, int ring_e, uint32_t off, uint32_t& it, const CUtensorMap* tm,
                  int row, int seq, uint64_t pol) -> bool {
    const uint32_t s = it & 1u;
    if (it >= 2 && !wait_bar(c, p, ring_e + s, ((it >> 1) - 1) & 1u)) return false;
    uint8_t* dst = c.sm + off + s * TILE;
    mbar_arrive_expect_tx(&c.bar[ring_f + s], TILE);
    tma_load_3d(dst, tm, &c.bar[ring_f + s], 0, row, seq, pol);
    tma_load_3d(dst + PLANE, tm, &c.bar[ring_f + s], 64, row, seq, pol);
    ++it;
    return true;
  };
  // Before leaving, wait (bounded) for every load still in flight so no TMA
  // write lands in shared memory after the CTA exits.
  auto drain = [&]() {
    const uint32_t rings[3][2] = {{B_QF, q_it}, {B_KF, k_it}, {B_VF, v_it}};
    for (int r = 0; r < 3; ++r)
      for (uint32_t j = rings[r][1] >= 2 ? rings[r][1] - 2 : 0; j < rings[r][1]; ++j)
        mbar_wait(&c.bar[rings[r][0] + (j & 1u)], (j >> 1) & 1u, p.wait_limit_ns);
  };
  for (;;) {
    const int w = next_work(p, static_next);
    const uint32_t ws = w_it & 1u;
    if (w_it >= 2 && !wait_bar(c, p, B_WE + ws, ((w_it >> 1) - 1) & 1u)) break;
    c.misc[1 + ws] = static_cast<uint32_t>(w);
    mbar_arrive(&c.bar[B_WF + ws]);
    ++w_it;
    if (w >= p.total) break;
    const Item it = decode_item(p, w);
    bool ok = true;
    if (it.phase1) {
      for (int b = 0; b < it.nb && ok; ++b) {
        const int row = it.t0 + b * BLK;
        ok = load(B_KF, B_KE, OFF_K, k_it, tk, row, it.seq, pol_last) &&
             load(B_VF, B_VE, OFF_V, v_it, tv, row, it.seq, pol_last);
      }
    }
    for (int n = 0; n < it.nb && ok; ++n) {
      const int row = it.t0 + n * BLK;
      ok = load(B_QF, B_QE, OFF_Q, q_it, tq, row, it.seq, pol_first) &&
           load(B_KF, B_KE, OFF_K, k_it, tk, row, it.seq, pol_first) &&
           load(B_VF, B_VE, OFF_V, v_it, tv, row, it.seq, pol_first);
    }
    if (!ok) break;
  }
  drain();
}

// ---------------------------------------------------------------------------
// MMA issuer: one thread issues every tcgen05.mma.
// ---------------------------------------------------------------------------
__device__ void mma_issue_loop(const Ctx& c, const Params& p) {
  constexpr uint32_t ID_KMAJ = idesc_bf16_f32(128, 128, false, false);  // Q K^T
  constexpr uint32_t ID_BMN = idesc_bf16_f32(128, 128, false, true);    // Q~ S, P V
  constexpr uint32_t ID_AMN = idesc_bf16_f32(128, 128, true, true);     // K~^T V
  const uint32_t sbase = smem_u32(c.sm);
  const uint32_t kvb = sbase + OFF_KVB;
  uint32_t q_it = 0, k_it = 0, v_it = 0, w_it = 0, gb = 0;
  uint32_t ready_n = 0, kvb_n = 0, kvfree_n = 0;
  uint32_t kt_n[2] = {0, 0};

  // S/P buffer (gb & 1) <- Q K^T for phase-2 block gidx of the current item.
  auto issue_S = [&](uint32_t qi, uint32_t ki, uint32_t gidx) -> bool {
    const uint32_t qs = qi & 1u, ks = ki & 1u, buf = gidx & 1u;
    if (!wait_bar(c, p, B_QF + qs, (qi >> 1) & 1u)) return false;
    if (!wait_bar(c, p, B_KF + ks, (ki >> 1) & 1u)) return false;
    if (gidx >= 2 && !wait_bar(c, p, B_SE + buf, ((gidx >> 1) - 1) & 1u)) return false;
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
    if (w >= p.total) return;
    const Item it = decode_item(p, w);
    if (!wait_bar(c, p, B_KV_FREE, kvfree_n++ & 1u)) return;
    if (it.phase1) {
      for (int b = 0; b < it.nb; ++b) {
        const uint32_t ks = k_it & 1u, vs = v_it & 1u;
        if (!wait_bar(c, p, B_KT + ks, kt_n[ks]++ & 1u)) return;
        if (!wait_bar(c, p, B_VF + vs, (v_it >> 1) & 1u)) return;
        tc_fence_after();
        const uint32_t ka = sbase + OFF_K + ks * TILE, va = sbase + OFF_V + vs * TILE;
#pragma unroll
        for (uint32_t kk = 0; kk < 8; ++kk)
          mma_ss(c.tmem + TM_KV, sdesc_sw128(ka + kk * 2048u, PLANE, 1024),
                 sdesc_sw128(va + kk * 2048u, PLANE, 1024), ID_AMN, (b > 0) || (kk > 0));
        mma_commit(&c.bar[B_KE + ks]);
        mma_commit(&c.bar[B_VE + vs]);
        ++k_it;
        ++v_it;
      }
      mma_commit(&c.bar[B_AGG_FULL]);
    }
    const uint32_t q0 = q_it, k0 = k_it, v0 = v_it, g0 = gb;
    const uint32_t nb = static_cast<uint32_t>(it.nb);
    if (!issue_S(q0, k0, g0)) return;
    for (uint32_t n = 0; n < nb; ++n) {
      const uint32_t g = g0 + n;
      const uint32_t qs = (q0 + n) & 1u, ks = (k0 + n) & 1u, vs = (v0 + n) & 1u;
      if (!wait_bar(c, p, B_READY, ready_n++ & 1u)) return;
      if (!wait_bar(c, p, B_KVB_READY, kvb_n++ & 1u)) return;
      if (!wait_bar(c, p, B_VF + vs, ((v0 + n) >> 1) & 1u)) return;
      tc_fence_after();
      const uint32_t qa = sbase + OFF_Q + qs * TILE, ka = sbase + OFF_K + ks * TILE;
      const uint32_t va = sbase + OFF_V + vs * TILE;
      // state += (decayed K)^T V
#pragma unroll
      for (uint32_t kk = 0; kk < 8; ++kk)
        mma_ss(c.tmem + TM_KV, sdesc_sw128(ka + kk * 2048u, PLANE, 1024),
               sdesc_sw128(va + kk * 2048u, PLANE, 1024), ID_AMN, 1);
      if (g >= 1 && !wait_bar(c, p, B_O_EMPTY, (g - 1) & 1u)) return;
      tc_fence_after();
      // O = (gamma^(i+1) Q) S_bf16
#pragma unroll
      for (uint32_t kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * PLANE + (kk & 3u) * 32u;
        mma_ss(c.tmem + TM_O, sdesc_sw128(qa + off, 16, 1024),
               sdesc_sw128(kvb + kk * 2048u, PLANE, 1024), ID_BMN, kk > 0);
      }
      // Q and K tiles are dead once the state update and the inter term finish.
      mma_commit(&c.bar[B_KVO_DONE]);
      mma_commit(&c.bar[B_QE + qs]);
      mma_commit(&c.bar[B_KE + ks]);
      // O += P V, P read from TMEM (bf16 pairs in the S buffer)
#pragma unroll
      for (uint32_t kk = 0; kk < 8; ++kk)
        mma_ts(c.tmem + TM_O, c.tmem + TM_S0 + (g & 1u) * 128u + kk * 8u,
               sdesc_sw128(va + kk * 2048u, PLANE, 1024), ID_BMN, 1);
      mma_commit(&c.bar[B_O_FULL]);
      mma_commit(&c.bar[B_SE + (g & 1u)]);
      // The V tile is released by the epilogue after it has staged the output there.
      if (n + 1 < nb && !issue_S(q0 + n + 1, k0 + n + 1, g + 1)) return;
    }
    q_it += nb;
    k_it += nb;
    v_it += nb;
    gb += nb;
  }
}

// Runs the issue loop, then waits (bounded) until every MMA it issued has
// completed, so TMEM is never released under a running MMA.
__device__ void mma_issuer(const Ctx& c, const Params& p) {
  mma_issue_loop(c, p);
  mma_commit(&c.bar[B_DRAIN]);
  mbar_wait(&c.bar[B_DRAIN], 0, p.wait_limit_ns);
}

// ---------------------------------------------------------------------------
// Compute warps (256 threads): thread owns TMEM lane / tile row r and the
// column half hf (64 columns) of that row.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_row64(const float* src, float* x) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 v = __ldcg(s4 + i);
    x[4 * i] = v.x;
    x[4 * i + 1] = v.y;
    x[4 * i + 2] = v.z;
    x[4 * i + 3] = v.w;
  }
}

__device__ __forceinline__ void store_row64(float* dst, const float* x) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 16; ++i)
    __stcg(d4 + i, make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]));
}

// Entering state of a work item: zero, the caller's initial state, or the
// inclusive state published by the previous chunk.  Returns false on failure.
__device__ bool entering_state(const Ctx& c, const Params& p, const Item& it, uint32_t tid,
                               int64_t row_off, uint32_t& csync_n, float* prev) {
  if (it.chunk > 0) {
    const int slot = (it.chunk - 1) & 1;
    if (tid == 0) {
      const int* flag = p.flags + it.seq * 2 + slot;
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while (ld_acquire_gpu(flag) != it.chunk) {
        if ((++spins & 15u) == 0 &&
            (aborted(c) || globaltimer_ns() - t0 > p.wait_limit_ns)) {
          fail(c, p, 2);
          break;
        }
      }
    }
    if (!csync(c, p, csync_n)) return false;
    load_row64(p.prefix + (static_cast<int64_t>(it.seq) * 2 + slot) * (HD * HD) + row_off, prev);
  } else if (p.init_state) {
    load_row64(p.init_state + static_cast<int64_t>(it.seq) * (HD * HD) + row_off, prev);
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i) prev[i] = 0.f;
  }
  return true;
}

__device__ void compute(const Ctx& c, const Params& p, const CUtensorMap* to) {
  const uint32_t tid = threadIdx.x;  // 0..255
  const uint32_t warp = tid >> 5;
  const uint32_t r = (warp & 3u) * 32u + (tid & 31u);
  const int ri = static_cast<int>(r);
  const uint32_t hf = warp >> 2;
  const uint32_t lane_base = ((warp & 3u) * 32u) << 16;
  const uint32_t t_kv = c.tmem + lane_base + TM_KV + hf * 64u;
  const uint32_t t_o = c.tmem + lane_base + TM_O + hf * 64u;
  const int64_t row_off = static_cast<int64_t>(r) * HD + hf * 64;
  const uint64_t pol_out = policy_evict_first();
  uint32_t q_it = 0, k_it = 0, v_it = 0, w_it = 0, gb = 0, agg_n = 0, csync_n = 0;
  // V slot whose staged output the last TMA stores may still read (thread 0)
  int pend_v = -1;
  auto release_pending = [&]() {
    if (tid == 0 && pend_v >= 0) {
      bulk_wait_group_read<0>();
      mbar_arrive(&c.bar[B_VE + pend_v]);
      pend_v = -1;
    }
  };

  bool ok = true;
  while (ok) {
    const uint32_t ws = w_it & 1u;
    if (!cwait(c, p, B_WF + ws, (w_it >> 1) & 1u)) break;
    const int w = static_cast<int>(c.misc[1 + ws]);
    mbar_arrive(&c.bar[B_WE + ws]);
    ++w_it;
    if (w >= p.total) break;
    const Item it = decode_item(p, w);
    const float lam = p.slopes[it.seq % p.H];

    if (!csync(c, p, csync_n)) break;  // the previous item's table is no longer read
    if (tid <= BLK) c.gpow[tid] = expf(-lam * static_cast<float>(tid));
    if (!csync(c, p, csync_n)) break;
    mbar_arrive(&c.bar[B_KV_FREE]);

    // ---- phase 1: local chunk state from decayed K ----
    if (it.phase1) {
      for (int b = 0; b < it.nb && ok; ++b) {
        const uint32_t ks = k_it & 1u;
        if (!cwait(c, p, B_KF + ks, (k_it >> 1) & 1u)) { ok = false; break; }
        const int jc = b * BLK + ri;
        const float f = jc < it.Lc ? expf(-lam * static_cast<float>(it.Lc - 1 - jc)) : 0.f;
        scale_row(c.sm + OFF_K + ks * TILE + hf * PLANE + r * 128u, r, f);
        fence_proxy_async_smem();
        mbar_arrive(&c.bar[B_KT + ks]);
        ++k_it;
        ++v_it;
      }
      if (!ok) break;
    }

    // ---- entering state; publication of this chunk's inclusive state ----
    {
      float prev[64];
      if (!entering_state(c, p, it, tid, row_off, csync_n, prev)) break;
      if (it.phase1) {
        if (!cwait(c, p, B_AGG_FULL, agg_n++ & 1u)) break;
        tc_fence_after();
        float agg[64];
        tmem_ld64(t_kv, agg);
        const float gL = expf(-lam * static_cast<float>(it.Lc));
#pragma unroll
        for (int i = 0; i < 64; ++i) agg[i] = fmaf(gL, prev[i], agg[i]);
        store_row64(p.prefix + (static_cast<int64_t>(it.seq) * 2 + (it.chunk & 1)) * (HD * HD) +
                        row_off,
                    agg);
        __threadfence();
        if (!csync(c, p, csync_n)) break;
        if (tid == 0) st_release_gpu(p.flags + it.seq * 2 + (it.chunk & 1), it.chunk + 1);
      }
      // state for block 0: bf16 copy for the MMA, fp32 copy decayed by gamma^len0
      store_row_bf16(c.sm + OFF_KVB + hf * PLANE + r * 128u, r, prev);
      tmem_st64(t_kv, prev, c.gpow[min(BLK, it.Lc)]);
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&c.bar[B_KVB_READY]);
    }

    // ---- phase 2: blocked form from the entering state ----
    for (int n = 0; n < it.nb; ++n) {
      const uint32_t g = gb;
      const int len = min(BLK, it.Lc - n * BLK);
      const uint32_t qs = q_it & 1u, ks = k_it & 1u, vs = v_it & 1u;
      uint8_t* qtile = c.sm + OFF_Q + qs * TILE;
      uint8_t* ktile = c.sm + OFF_K + ks * TILE;
      uint8_t* vtile = c.sm + OFF_V + vs * TILE;
      const uint32_t t_s = c.tmem + lane_base + TM_S0 + (g & 1u) * 128u;

      // (A) decay-causal mask of Q K^T into P (bf16, TMEM); gamma^(i+1) Q and
      //     gamma^(len-1-j) K in place in shared memory.
      if (!cwait(c, p, B_SF + (g & 1u), (g >> 1) & 1u) ||
          !cwait(c, p, B_QF + qs, (q_it >> 1) & 1u) ||
          !cwait(c, p, B_KF + ks, (k_it >> 1) & 1u)) { ok = false; break; }
      tc_fence_after();
      {
        float sv[64];
        tmem_ld64(t_s + hf * 64u, sv);
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j0 = static_cast<int>(hf) * 64 + 2 * i;
          const float p0 = (j0 <= ri && ri < len) ? sv[2 * i] * c.gpow[ri - j0] : 0.f;
          const float p1 = (j0 + 1 <= ri && ri < len) ? sv[2 * i + 1] * c.gpow[ri - j0 - 1] : 0.f;
          pk[i] = pack_bf16x2(p0, p1);
        }
        // every S column is in registers before P (half as many columns) overwrites it
        if (!csync(c, p, csync_n)) { ok = false; break; }
        tmem_st32(t_s + hf * 32u, pk);
      }
      scale_row(qtile + hf * PLANE + r * 128u, r, ri < len ? c.gpow[ri + 1] : 0.f);
      scale_row(ktile + hf * PLANE + r * 128u, r, ri < len ? c.gpow[len - 1 - ri] : 0.f);
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&c.bar[B_READY]);
      release_pending();

      // (B) state: bf16 copy for the next block's inter term, then decay in TMEM
      if (!cwait(c, p, B_KVO_DONE, g & 1u)) { ok = false; break; }
      tc_fence_after();
      {
        float kv[64];
        tmem_ld64(t_kv, kv);
        if (n + 1 < it.nb) {
          store_row_bf16(c.sm + OFF_KVB + hf * PLANE + r * 128u, r, kv);
          tmem_st64(t_kv, kv, c.gpow[min(BLK, it.Lc - (n + 1) * BLK)]);
          fence_proxy_async_smem();
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&c.bar[B_KVB_READY]);
        } else if (p.final_state && it.chunk + 1 == p.nchunks) {
          store_row64(p.final_state + static_cast<int64_t>(it.seq) * (HD * HD) + row_off, kv);
        }
      }

      // (C) epilogue: O -> swizzled staging in this block's V slot (dead once O
      //     is complete), 64 columns at a time -> TMA store.
      if (!cwait(c, p, B_O_FULL, g & 1u)) { ok = false; break; }
      tc_fence_after();
      {
        float o[64];
        tmem_ld64(t_o, o);
        tc_fence_before();
        mbar_arrive(&c.bar[B_O_EMPTY]);
        const int row = it.t0 + n * BLK;
        for (uint32_t half = 0; half < 2 && ok; ++half) {
          if (hf == half) {
            store_row_f32(vtile + r * 128u, r, o);
            store_row_f32(vtile + PLANE + r * 128u, r, o + 32);
          }
          fence_proxy_async_smem();
          if (!csync(c, p, csync_n)) { ok = false; break; }
          if (tid == 0) {
            tma_store_3d(to, vtile, 64 * half, row, it.seq, pol_out);
            tma_store_3d(to, vtile + PLANE, 64 * half + 32, row, it.seq, pol_out);
            bulk_commit_group();
            if (half == 0) bulk_wait_group_read<0>();
          }
          if (half == 0 && !csync(c, p, csync_n)) { ok = false; break; }
        }
        if (tid == 0) pend_v = static_cast<int>(vs);
      }
      if (!ok) break;
      ++q_it;
      ++k_it;
      ++v_it;
      ++gb;
    }
    release_pending();
  }
  if (tid == 0) bulk_wait_group<0>();
}

__global__ void __launch_bounds__(THREADS, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Ctx c;
  c.sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
  c.bar = reinterpret_cast<uint64_t*>(c.sm + OFF_BAR);
  c.gpow = reinterpret_cast<float*>(c.sm + OFF_GPOW);
  c.misc = reinterpret_cast<volatile uint32_t*>(c.sm + OFF_MISC);
  const uint32_t warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.bar[B_QF + i], 1);
      mbar_init(&c.bar[B_QE + i], 1);
      mbar_init(&c.bar[B_KF + i], 1);
      mbar_init(&c.bar[B_KE + i], 1);
      mbar_init(&c.bar[B_VF + i], 1);
      mbar_init(&c.bar[B_VE + i], 1);
      mbar_init(&c.bar[B_SF + i], 1);
      mbar_init(&c.bar[B_SE + i], 1);
      mbar_init(&c.bar[B_WF + i], 1);
      mbar_init(&c.bar[B_WE + i], 1 + C_THREADS);
      mbar_init(&c.bar[B_KT + i], C_THREADS);
    }
    mbar_init(&c.bar[B_READY], C_THREADS);
    mbar_init(&c.bar[B_KVB_READY], C_THREADS);
    mbar_init(&c.bar[B_KVO_DONE], 1);
    mbar_init(&c.bar[B_O_FULL], 1);
    mbar_init(&c.bar[B_O_EMPTY], C_THREADS);
    mbar_init(&c.bar[B_AGG_FULL], 1);
    mbar_init(&c.bar[B_KV_FREE], C_THREADS);
    mbar_init(&c.bar[B_CSYNC], C_THREADS);
    mbar_init(&c.bar[B_DRAIN], 1);
    c.misc[3] = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(const_cast<uint32_t*>(&c.misc[0]), 512);
    tmem_relinquish();
  }
  if (warp == PRODUCER_WARP && lane_id() == 0) {
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    prefetch_tmap(&to);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  c.tmem = c.misc[0];

  if (warp == PRODUCER_WARP) {
    if (lane_id() == 0) producer(c, p, &tq, &tk, &tv);
  } else if (warp == MMA_WARP) {
    if (lane_id() == 0) mma_issuer(c, p);
    __syncwarp();
  } else {
    compute(c, p, &to);
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
