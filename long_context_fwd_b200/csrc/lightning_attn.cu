// lightning_attn.cu -- C ABI of the library: argument checks, TMA tensor maps,
// scratch for the chunked scan, and kernel launches.  Every compute step runs
// in the kernels included below; the host code only marshals and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <chrono>
#include <random>

#include "lightning_attn.h"
#include "sm100_ptx.cuh"
#include "tmap.h"

namespace la {
// Sticky device-side status word: bit 0 = an mbarrier wait ran out of time,
// bit 1 = a chunk-scan flag wait ran out of time, bit 2 = a split-scan share
// or chain exceeded its shared-memory list (excluded by the host's plan).
__device__ int g_status;
}  // namespace la

#include "la_decode.cuh"
#include "la_fwd_f32.cuh"
#include "la_fwd_sm100.cuh"
#include "la_state.cuh"

namespace {

constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s per device-side wait

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

inline bool dims_ok(int B, int H, int N, int D, int E) {
  if (B < 1 || H < 1 || N < 1) return false;
  const __int128 n = static_cast<__int128>(B) * H * N * (D > E ? D : E);
  return n < (static_cast<__int128>(1) << 62) && static_cast<long long>(B) * H < (1ll << 31);
}

// Text of the CUDA error behind the calling thread's last LA_ERR_CUDA.
thread_local const char* t_last_cuda_error = "no error";

inline int cuda_fail(cudaError_t e) {
  t_last_cuda_error = cudaGetErrorString(e);
  return LA_ERR_CUDA;
}

inline int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LA_OK : cuda_fail(e);
}

inline int* status_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, la::g_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 148;
  return n;
}

// Caller's cap on the prefill kernel's persistent grid (0 = none), shared by
// every thread of the process (lightning_attn_set_cta_limit).
std::atomic<int> g_cta_limit{0};

// The prefill kernel takes two sets of q, k, v, out tensor maps: the second is
// role 1's in a paired launch (a copy of the first otherwise).
using FwdKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           const CUtensorMap, const CUtensorMap, const CUtensorMap,
                           const CUtensorMap, const CUtensorMap, const la::fwd::Params);

FwdKernel pick_fwd_kernel(int rank, bool rev, bool fused) {
  using la::fwd::fwd_bf16_kernel;
  if (fused) return rank == 3 ? fwd_bf16_kernel<3, false, true> : fwd_bf16_kernel<4, false, true>;
  return rank == 3 ? (rev ? fwd_bf16_kernel<3, true, false> : fwd_bf16_kernel<3, false, false>)
                   : (rev ? fwd_bf16_kernel<4, true, false> : fwd_bf16_kernel<4, false, false>);
}

// Sets the kernel's shared-memory attribute (it belongs to the current
// device's context, so on every call) and returns in *ctas how many of its
// CTAs can be resident at once on the current device: SMs x CTAs per SM (one,
// by design), capped by the caller's limit.  The static work splits plan for
// exactly that many CTAs and are launched cooperatively, so that either all
// of them run at the same time or the launch fails up front.
int prepare_fwd_kernel(FwdKernel kern, int* ctas) {
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, la::fwd::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e);
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, la::fwd::THREADS,
                                                    la::fwd::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e);
  if (per_sm < 1) return LA_ERR_UNSUPPORTED;
  long long n = static_cast<long long>(per_sm) * sm_count();
  const int cap = g_cta_limit.load(std::memory_order_relaxed);
  if (cap > 0 && cap < n) n = cap;
  *ctas = static_cast<int>(n < (1 << 20) ? n : (1 << 20));
  return LA_OK;
}

// How the (b, h) sequences become work items for the persistent grid.
//  * At least as many sequences as SMs: a balanced hand-over split.  Each CTA
//    gets the same number of 128-token blocks of the concatenated sequences; a
//    sequence that crosses a CTA boundary is handed over through its final
//    state (no extra pass), and the two CTAs order their work so that the
//    hand-over is not waited for.  Without this, 256 sequences on 148 SMs
//    would take two full waves with 40 SMs idle in the second.
//  * Fewer sequences than SMs (at least SMs/8 of them, and more than 8 blocks
//    each): a split scan.  Each of nseq CTAs computes the last T/G blocks of
//    one sequence (T blocks in all, G CTAs); the other G - nseq CTAs share the
//    first parts equally.  Every share but a sequence's first needs the state
//    at its start, so a local-state pass over the first parts (an extra read of
//    their K and V, shared equally by all CTAs) runs first; entering states
//    chain the published local states.  The extra pass covers 1 - nseq/G of
//    the tokens (57% for 64 sequences) instead of nearly all of them.
//  * Otherwise (a handful of long sequences): a parallel scan over chunks of
//    2048-8192 tokens (measured sweet spot on B200) handed out by an atomic
//    ticket; every chunk but the last computes its local state first.
//  * An explicit chunk length shorter than N always selects the chunk scan.
struct Plan {
  int L = 0, nchunks = 1, mode = 0, grid = 0;
  int nblk = 0, F = 0, G2 = 0;
  long long P = 0, total = 0;
  size_t ctrl = 0, bytes = 0;  // scratch: ticket + flags, then 64 KiB chunk states
};

// Scratch control block: the ticket (padded to 8 bytes), then n 64-bit flags.
size_t ctrl_bytes(size_t n_flags) { return (8 + n_flags * 8 + 255) / 256 * 256; }

Plan make_plan(int nseq, int N, int sms, int chunk) {
  Plan pl;
  const int nblk = (N + 127) / 128;
  pl.nblk = nblk;
  const size_t state_bytes = 128 * 128 * sizeof(float);
  if (chunk == 0 && nseq >= sms) {
    pl.mode = la::fwd::MODE_HANDOVER;
    pl.L = nblk * 128;
    pl.grid = sms;
    if (nseq % sms != 0) {  // some sequence crosses a CTA boundary
      pl.ctrl = ctrl_bytes(static_cast<size_t>(sms));
      pl.bytes = pl.ctrl + static_cast<size_t>(sms) * state_bytes;
    }
    return pl;
  }
  if (chunk == 0 && nblk > 8 && 8 * nseq >= sms) {
    // tail = blocks of each sequence's last share, about T/G; of the two
    // roundings take the one whose longest share (outputs + the local-state
    // pass at ~0.4 of the cost per block) is shorter, and use the split only
    // if that beats one whole sequence per SM
    const long long T = static_cast<long long>(nseq) * nblk;
    const long long G2 = sms - nseq;
    double best = static_cast<double>(nblk);
    long long best_tail = 0;
    for (long long tail = T / sms; tail <= (T + sms - 1) / sms; ++tail) {
      const long long F = nblk - tail, P = static_cast<long long>(nseq) * F;
      if (tail < 1 || F < 1 || P >= (1ll << 31)) continue;
      const long long packed = (P + G2 - 1) / G2;
      const double span = static_cast<double>(tail > packed ? tail : packed) +
                          0.4 * static_cast<double>((P + sms - 1) / sms);
      if (span < best) {
        best = span;
        best_tail = tail;
      }
    }
    if (best_tail > 0) {
      const long long F = nblk - best_tail;
      pl.mode = la::fwd::MODE_SPLIT_SCAN;
      pl.L = nblk * 128;
      pl.grid = sms;
      pl.F = static_cast<int>(F);
      pl.G2 = static_cast<int>(G2);
      pl.P = static_cast<long long>(nseq) * F;
      pl.ctrl = ctrl_bytes(2 * static_cast<size_t>(sms));
      pl.bytes = pl.ctrl + 2 * static_cast<size_t>(sms) * state_bytes;
      return pl;
    }
  }
  int L = chunk;
  if (L == 0) {
    L = nblk * 128;
    if (nblk > 8) {
      const int want_chunks = (4 * sms + nseq - 1) / nseq;
      L = ((N + want_chunks - 1) / want_chunks + 127) / 128 * 128;
      if (L < 2048) L = 2048;
      if (L > 8192) L = 8192;
    }
  }
  if (L > nblk * 128) L = nblk * 128;
  pl.L = L;
  pl.nchunks = (N + L - 1) / L;
  pl.total = static_cast<long long>(nseq) * pl.nchunks;
  pl.grid = static_cast<int>(pl.total < sms ? pl.total : sms);
  if (pl.nchunks > 1) {
    pl.ctrl = ctrl_bytes(static_cast<size_t>(nseq) * 2);
    pl.bytes = pl.ctrl + static_cast<size_t>(nseq) * 2 * state_bytes;
  }
  return pl;
}

// The state pass (lightning_attn_state): every chunk a local-state item of the
// ticketed chunk scan, the last one of each sequence writing the caller's
// final state.  Whole sequences when there are enough of them to fill the
// grid; otherwise chunks of 1024-8192 tokens, about four items per CTA.
Plan make_state_plan(int nseq, int N, int sms, int chunk) {
  Plan pl;
  const int nblk = (N + 127) / 128;
  pl.nblk = nblk;
  pl.mode = la::fwd::MODE_TICKETS;
  int L = chunk;
  if (L == 0) {
    L = nblk * 128;
    if (nseq < sms && nblk > 8) {
      const int want_chunks = (4 * sms + nseq - 1) / nseq;
      L = ((N + want_chunks - 1) / want_chunks + 127) / 128 * 128;
      if (L < 1024) L = 1024;
      if (L > 8192) L = 8192;
    }
  }
  if (L > nblk * 128) L = nblk * 128;
  pl.L = L;
  pl.nchunks = (N + L - 1) / L;
  pl.total = static_cast<long long>(nseq) * pl.nchunks;
  pl.grid = static_cast<int>(pl.total < sms ? pl.total : sms);
  if (pl.nchunks > 1) {
    const size_t state_bytes = 128 * 128 * sizeof(float);
    pl.ctrl = ctrl_bytes(static_cast<size_t>(nseq) * 2);
    pl.bytes = pl.ctrl + static_cast<size_t>(nseq) * 2 * state_bytes;
  }
  return pl;
}

// Fills the launch parameters that depend on the plan.
void apply_plan(const Plan& pl, int nseq, la::fwd::Params& p) {
  p.nseq = nseq;
  p.L = pl.L;
  p.nchunks = pl.nchunks;
  p.total = static_cast<int>(pl.total);
  p.mode = pl.mode;
  p.nblk = pl.nblk;
  p.F = pl.F;
  p.G2 = pl.G2;
  p.P = pl.P;
}

void set_scratch(const Plan& pl, void* scratch, la::fwd::Params& p) {
  p.ticket = static_cast<int*>(scratch);
  p.flags = reinterpret_cast<unsigned long long*>(static_cast<char*>(scratch) + 8);
  p.prefix = reinterpret_cast<float*>(static_cast<char*>(scratch) + pl.ctrl);
}

// Only the chunk scan's ticket and flags (chunk numbers) need zeroing before a
// launch; the hand-over and the split scan publish the launch's tag -- except
// in a stream capture, where the tag is frozen into the graph and every replay
// would find the previous replay's flags already set: there the captured
// memset clears them (a zero flag never equals a tag).
bool needs_zeroed_ctrl(const Plan& pl, cudaStream_t stream) {
  if (pl.mode == la::fwd::MODE_TICKETS) return true;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  return cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
}

// A nonzero 64-bit value unique to each launch of this process: the flag value
// the hand-over and the split scan publish, so that scratch left by earlier
// launches (or holding anything else) never reads as published.  SplitMix64
// (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
// OOPSLA 2014) of a per-process counter times an odd constant plus a random
// seed: a bijection of the counter, so no two launches share a tag, and other
// contents of the scratch match it with probability 2^-64 per flag read.
unsigned long long launch_tag() {
  static const unsigned long long seed = [] {
    // the C ABI never throws: without an entropy source, the clock and an
    // address of this process seed it (distinct launches still get distinct
    // tags; only foreign scratch contents would be less unpredictable)
    unsigned long long z = static_cast<unsigned long long>(
        std::chrono::high_resolution_clock::now().time_since_epoch().count());
    z ^= reinterpret_cast<uintptr_t>(&z);
    try {
      std::random_device rd;
      z ^= (static_cast<unsigned long long>(rd()) << 32) ^ rd();
    } catch (...) {
    }
    return z;
  }();
  static std::atomic<unsigned long long> counter{0};
  for (;;) {
    unsigned long long z = seed + 0x9E3779B97F4A7C15ull * (counter.fetch_add(1) + 1);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    if (z != 0) return z;
  }
}

// Element strides {b, h, t} of q, k, v, out and the fused layer's gate (d or e
// contiguous).
struct Strides {
  long long s[5][3];
};

Strides contiguous_strides(int H, int N, int D, int E) {
  Strides st;
  const long long w[5] = {D, D, E, E, E};
  for (int i = 0; i < 5; ++i) {
    st.s[i][2] = w[i];
    st.s[i][1] = static_cast<long long>(N) * w[i];
    st.s[i][0] = static_cast<long long>(H) * N * w[i];
  }
  return st;
}

// TMA needs every stride in bytes to be a multiple of 16 and below 2^40 (the
// gate's rows are read with 16-byte copies, which need the same).
bool strides_ok(const Strides& st, bool out_bf16) {
  const int eb[5] = {2, 2, 2, out_bf16 ? 2 : 4, 2};
  for (int i = 0; i < 5; ++i)
    for (int j = 0; j < 3; ++j) {
      const long long b = st.s[i][j] * eb[i];
      if (st.s[i][j] < 0 || b % 16 != 0 || b >= (1ll << 40)) return false;
    }
  return true;
}

// The four tensor maps of the bf16 prefill: 3-D [B*H][N][cols] maps when
// every tensor is contiguous head-major, else 4-D maps (p.cslot says where t,
// h and b went).  *rank receives 3 or 4.
bool build_maps(const void* q, const void* k, const void* v, const void* out, int B, int H, int N,
                int D, int E, const Strides& st, CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv,
                CUtensorMap* to, la::fwd::Params& p, int* rank, bool out_bf16 = false) {
  // Column extents D and E: a 64-wide tensor leaves the second 64-column half
  // of every 128-wide tile outside the map, so TMA fills it with zeros (no
  // memory traffic) and clips stores there; zero columns add nothing to any
  // product, so the 128 x 128 kernel computes the D x E result exactly.
  p.D = D;
  p.E = E;
  const Strides cont = contiguous_strides(H, N, D, E);
  bool contiguous = true;
  for (int i = 0; i < 4; ++i)  // q, k, v, out (the gate is read without a map)
    for (int j = 0; j < 3; ++j) {
      const bool unused = (j == 0 && B == 1) || (j == 1 && H == 1);  // extent-1 dimension
      contiguous = contiguous && (unused || st.s[i][j] == cont.s[i][j]);
    }
  if (contiguous) {
    *rank = 3;
    const uint64_t nseq = static_cast<uint64_t>(B) * H;
    return la::make_tmap_3d(tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, N, nseq, 64, 128) &&
           la::make_tmap_3d(tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, N, nseq, 64, 128) &&
           la::make_tmap_3d(tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, N, nseq, 64, 128) &&
           (out_bf16 ? la::make_tmap_3d(to, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, N, nseq, 64, 128)
                     : la::make_tmap_3d(to, out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, E, N, nseq, 32, 128));
  }
  *rank = 4;
  const uint64_t ext[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(H),
                           static_cast<uint64_t>(B)};
  CUtensorMap* maps[4] = {tq, tk, tv, to};
  const void* bases[4] = {q, k, v, out};
  for (int i = 0; i < 4; ++i) {
    const uint64_t str[3] = {static_cast<uint64_t>(st.s[i][2]), static_cast<uint64_t>(st.s[i][1]),
                             static_cast<uint64_t>(st.s[i][0])};
    const bool f32 = i == 3 && !out_bf16;
    if (!la::make_tmap_4d(maps[i], bases[i],
                          f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          f32 ? 4 : 2, i < 2 ? D : E, ext, str, f32 ? 32 : 64, 128, &p.cslot[i]))
      return false;
  }
  return true;
}

// Launches the prefill kernel.  The hand-over and the split scan have CTAs
// that wait for states other CTAs publish, so those launches are cooperative:
// the runtime then starts the grid only with every CTA resident (or fails the
// launch) instead of leaving a waiting CTA on an SM that a CTA it waits for
// needs.  The chunk scan hands work out by ticket in order and needs no such
// guarantee.
// role1: the second role's four maps (q, k, v, out) of a paired launch, or null.
int launch_fwd(FwdKernel kern, int grid, bool cooperative, cudaStream_t stream,
               const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const CUtensorMap& to, const la::fwd::Params& p,
               const CUtensorMap* role1 = nullptr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(la::fwd::THREADS);
  cfg.dynamicSmemBytes = la::fwd::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 1 : 0;
  const cudaError_t e =
      role1 ? cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, role1[0], role1[1], role1[2], role1[3], p)
            : cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, tq, tk, tv, to, p);
  if (e != cudaSuccess) return cuda_fail(e);
  return launch_status();
}

// The fused layer's extra operands (lightning_attn_fwd_fused).
struct FusedArgs {
  const void* gate;
  const float* norm_w;
  float eps;
};

int fwd_bf16_impl(const void* q, const void* k, const void* v, const float* slopes,
                  const float* init_state, float* final_state, void* out, int B, int H, int N,
                  int D, int E, int chunk, void* stream_ptr, const Strides* strides = nullptr,
                  bool reverse = false, int first_chunk = 0,
                  unsigned long long wait_limit_ns = kWaitLimitNs,
                  const FusedArgs* fused = nullptr) {
  if (!q || !k || !v || !slopes || !out) return LA_ERR_NULL;
  if (fused) {
    if (!fused->gate || !fused->norm_w) return LA_ERR_NULL;
    if (!aligned16(fused->gate) || !aligned16(fused->norm_w)) return LA_ERR_ALIGN;
    if (!(fused->eps >= 0.f) || fused->eps > 3.0e38f) return LA_ERR_SHAPE;
    if (reverse) return LA_ERR_UNSUPPORTED;
  }
  if (!dims_ok(B, H, N, D, E)) return LA_ERR_SHAPE;
  if ((D != 64 && D != 128) || (E != 64 && E != 128)) return LA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(slopes) ||
      (init_state && !aligned16(init_state)) || (final_state && !aligned16(final_state)))
    return LA_ERR_ALIGN;
  if (chunk < 0 || (chunk % 128) != 0) return LA_ERR_SHAPE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int nseq = B * H;

  const Strides st = strides ? *strides : contiguous_strides(H, N, D, E);
  if (!strides_ok(st, fused != nullptr)) return LA_ERR_ALIGN;
  la::fwd::Params p{};
  CUtensorMap tq, tk, tv, to;
  int rank = 3;
  if (!build_maps(q, k, v, out, B, H, N, D, E, st, &tq, &tk, &tv, &to, p, &rank,
                  fused != nullptr))
    return LA_ERR_CUDA;
  const FwdKernel kern = pick_fwd_kernel(rank, reverse, fused != nullptr);
  int ctas = 0;
  int rc = prepare_fwd_kernel(kern, &ctas);
  if (rc != LA_OK) return rc;
  const Plan pl = make_plan(nseq, N, ctas, chunk);
  if (pl.total >= (1ll << 31)) return LA_ERR_SHAPE;
  p.out = fused ? nullptr : static_cast<float*>(out);
  if (fused) {
    p.gate = static_cast<const uint16_t*>(fused->gate);
    p.norm_w = fused->norm_w;
    p.eps = fused->eps;
    for (int j = 0; j < 3; ++j) p.gstride[j] = st.s[4][j];
  }
  for (int j = 0; j < 3; ++j) p.ostride[j] = st.s[3][j];

  p.slopes = slopes;
  p.init_state = init_state;
  p.final_state = final_state;
  p.status = status_word();
  if (!p.status) return LA_ERR_CUDA;
  p.H = H;
  p.N = N;
  apply_plan(pl, nseq, p);
  p.ticket_base = first_chunk * nseq;
  p.wait_limit_ns = wait_limit_ns;

  p.tag = launch_tag();

  void* scratch = nullptr;
  if (pl.bytes) {
    cudaError_t e = cudaMallocAsync(&scratch, pl.bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    if (needs_zeroed_ctrl(pl, stream)) {
      e = cudaMemsetAsync(scratch, 0, pl.ctrl, stream);
      if (e != cudaSuccess) {
        cudaFreeAsync(scratch, stream);
        return cuda_fail(e);
      }
    }
    set_scratch(pl, scratch, p);
  }

  rc = launch_fwd(kern, pl.grid, pl.mode != la::fwd::MODE_TICKETS, stream, tq, tk, tv, to, p);
  if (scratch) {
    const cudaError_t e = cudaFreeAsync(scratch, stream);
    if (e != cudaSuccess && rc == LA_OK) rc = cuda_fail(e);
  }
  return rc;
}

// ---------------------------------------------------------------------------
// Allocation-free prefill: the chunk-scan scratch lives in a fixed device array.
// ---------------------------------------------------------------------------
// In host code the array's name is only a host-side stand-in: its device
// address in the current device's context is looked up with
// cudaGetSymbolAddress on every call (a table lookup once the library's device
// code is loaded, which the first call on each device does), so a context that
// was reset and re-created never gets a stale address.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

int noalloc_scratch_ptr(void** out) {
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  *out = ptr;
  return LA_OK;
}

int fwd_bf16_noalloc_impl(const void* q, const void* k, const void* v, const float* slopes,
                          float* out, int B, int H, int N, int D, int E, int chunk,
                          void* stream_ptr) {
  if (!q || !k || !v || !slopes || !out) return LA_ERR_NULL;
  if (!dims_ok(B, H, N, D, E)) return LA_ERR_SHAPE;
  if ((D != 64 && D != 128) || (E != 64 && E != 128)) return LA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(slopes))
    return LA_ERR_ALIGN;
  if (chunk < 0 || (chunk % 128) != 0) return LA_ERR_SHAPE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int nseq = B * H;
  // an explicit chunk length's scratch (two states per sequence) does not
  // depend on the grid: rejected on the host before touching the device
  if (chunk > 0 && make_plan(nseq, N, 1, chunk).bytes > LA_NOALLOC_SCRATCH_BYTES)
    return LA_ERR_WORKSPACE;
  const FwdKernel kern = pick_fwd_kernel(3, false, false);
  int sms = 0;
  const int prc = prepare_fwd_kernel(kern, &sms);
  if (prc != LA_OK) return prc;
  Plan pl = make_plan(nseq, N, sms, chunk);
  if (pl.mode != la::fwd::MODE_TICKETS && pl.bytes > LA_NOALLOC_SCRATCH_BYTES) {
    // a GPU with so many SMs that the chunk states do not fit: whole sequences
    pl = Plan{};
    pl.L = (N + 127) / 128 * 128;
    pl.nblk = (N + 127) / 128;
    pl.total = nseq;
    pl.grid = nseq < sms ? nseq : sms;
  }
  if (pl.total >= (1ll << 31)) return LA_ERR_SHAPE;
  if (pl.bytes > LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_WORKSPACE;

  la::fwd::Params p{};
  CUtensorMap tq, tk, tv, to;
  int rank = 3;
  const Strides st = contiguous_strides(H, N, D, E);
  if (!build_maps(q, k, v, out, B, H, N, D, E, st, &tq, &tk, &tv, &to, p, &rank))
    return LA_ERR_CUDA;
  p.out = out;
  for (int j = 0; j < 3; ++j) p.ostride[j] = st.s[3][j];

  p.slopes = slopes;
  p.status = status_word();
  if (!p.status) return LA_ERR_CUDA;
  p.H = H;
  p.N = N;
  apply_plan(pl, nseq, p);
  p.wait_limit_ns = kWaitLimitNs;
  p.tag = launch_tag();
  if (pl.bytes) {
    void* scratch = nullptr;
    const int rc = noalloc_scratch_ptr(&scratch);
    if (rc != LA_OK) return rc;
    // the array keeps the previous call's contents: the chunk scan's ticket
    // and flags must start at zero (the chunk states are always written
    // before they are read; the other splits' flags carry this launch's tag)
    if (needs_zeroed_ctrl(pl, stream)) {
      const cudaError_t e = cudaMemsetAsync(scratch, 0, pl.ctrl, stream);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    set_scratch(pl, scratch, p);
  }
  return launch_fwd(kern, pl.grid, pl.mode != la::fwd::MODE_TICKETS, stream, tq, tk, tv, to, p);
}

template <int D, int E>
int launch_f32(const float* q, const float* k, const float* v, const float* slopes, float* out,
               int B, int H, int N, cudaStream_t stream) {
  constexpr size_t smem = la::fwd_f32_smem_bytes<D, E>();
  const cudaError_t attr =
      cudaFuncSetAttribute(la::fwd_f32_kernel<D, E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (attr != cudaSuccess) return cuda_fail(attr);
  la::fwd_f32_kernel<D, E><<<B * H, 256, smem, stream>>>(q, k, v, slopes, out, H, N);
  return launch_status();
}

template <int D, int E>
int launch_decode(const void* q, const void* k, const void* v, float* state, const float* slopes,
                  float* out, int B, int H, cudaStream_t stream) {
  la::decode_kernel<D, E><<<B * H, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), state, slopes, out, H);
  return launch_status();
}

int state_impl(const void* k, const void* v, const float* slopes, const float* init_state,
               float* final_state, int B, int H, int N, int D, int E, int chunk,
               void* stream_ptr) {
  if (!k || !v || !slopes || !final_state) return LA_ERR_NULL;
  if (!dims_ok(B, H, N, D, E)) return LA_ERR_SHAPE;
  if ((D != 64 && D != 128) || (E != 64 && E != 128)) return LA_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(v) || !aligned4(slopes) || !aligned16(final_state) ||
      (init_state && !aligned16(init_state)))
    return LA_ERR_ALIGN;
  if (chunk < 0 || (chunk % 128) != 0) return LA_ERR_SHAPE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int nseq = B * H;
  la::fwd::Params p{};
  CUtensorMap tk, tv;
  const uint64_t ns = static_cast<uint64_t>(nseq);
  if (!la::make_tmap_3d(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, N, ns, 64, 128) ||
      !la::make_tmap_3d(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, N, ns, 64, 128))
    return LA_ERR_CUDA;
  p.D = D;
  p.E = E;
  const FwdKernel kern = pick_fwd_kernel(3, false, false);
  int ctas = 0;
  int rc = prepare_fwd_kernel(kern, &ctas);
  if (rc != LA_OK) return rc;
  const Plan pl = make_state_plan(nseq, N, ctas, chunk);
  if (pl.total >= (1ll << 31)) return LA_ERR_SHAPE;
  p.slopes = slopes;
  p.init_state = init_state;
  p.final_state = final_state;
  p.state_only = 1;
  p.status = status_word();
  if (!p.status) return LA_ERR_CUDA;
  p.H = H;
  p.N = N;
  apply_plan(pl, nseq, p);
  p.wait_limit_ns = kWaitLimitNs;
  p.tag = launch_tag();
  void* scratch = nullptr;
  if (pl.bytes) {
    cudaError_t e = cudaMallocAsync(&scratch, pl.bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemsetAsync(scratch, 0, pl.ctrl, stream);  // the ticket and chunk flags
    if (e != cudaSuccess) {
      cudaFreeAsync(scratch, stream);
      return cuda_fail(e);
    }
    set_scratch(pl, scratch, p);
  }
  // q and out take no part in the state pass: the K map stands in for both
  rc = launch_fwd(kern, pl.grid, false, stream, tk, tk, tv, tk, p);
  if (scratch) {
    const cudaError_t e = cudaFreeAsync(scratch, stream);
    if (e != cudaSuccess && rc == LA_OK) rc = cuda_fail(e);
  }
  return rc;
}

template <int D, int E>
int launch_decode_layer(const la::DecodeLayerArgs& a, int64_t nbh, cudaStream_t stream) {
  la::decode_layer_kernel<D, E><<<static_cast<unsigned>(nbh), 256, 0, stream>>>(a);
  return launch_status();
}

}  // namespace

extern "C" {

int lightning_attn_fwd(const void* q, const void* k, const void* v, const float* slopes,
                       float* out, int B, int H, int N, int D, int E, void* stream) {
  return fwd_bf16_impl(q, k, v, slopes, nullptr, nullptr, out, B, H, N, D, E, 0, stream);
}

int lightning_attn_fwd_ex(const void* q, const void* k, const void* v, const float* slopes,
                          const float* init_state, float* final_state, float* out, int B, int H,
                          int N, int D, int E, int chunk, void* stream) {
  return fwd_bf16_impl(q, k, v, slopes, init_state, final_state, out, B, H, N, D, E, chunk,
                       stream);
}

int lightning_attn_fwd_strided(const void* q, const void* k, const void* v, const float* slopes,
                               const float* init_state, float* final_state, float* out, int B,
                               int H, int N, int D, int E, const long long* q_strides,
                               const long long* k_strides, const long long* v_strides,
                               const long long* out_strides, int chunk, void* stream) {
  if (!q_strides || !k_strides || !v_strides || !out_strides) return LA_ERR_NULL;
  Strides st = {};  // (the gate's entry is not used)
  const long long* src[4] = {q_strides, k_strides, v_strides, out_strides};
  for (int i = 0; i < 4; ++i)
    for (int j = 0; j < 3; ++j) st.s[i][j] = src[i][j];
  return fwd_bf16_impl(q, k, v, slopes, init_state, final_state, out, B, H, N, D, E, chunk,
                       stream, &st);
}

int lightning_attn_fwd_anticausal(const void* q, const void* k, const void* v, const float* slopes,
                                  const float* init_state, float* final_state, float* out, int B,
                                  int H, int N, int D, int E, int chunk, void* stream) {
  return fwd_bf16_impl(q, k, v, slopes, init_state, final_state, out, B, H, N, D, E, chunk,
                       stream, nullptr, /*reverse=*/true);
}

// dk and dv in one launch.  Both are anti-causal operators that read q and
// dout (dk on (v, dout, q), dv on (k, q, dout)), so CTA 2j computes dk and CTA
// 2j + 1 dv of the same work items, planned for half the CTAs: the two CTAs
// of a pair stream the same q and dout tiles at about the same time, and the
// second read of each comes from L2.  Each role has its own scratch (ticket,
// flags, hand-over states).  Needs D == E and at least two CTAs; *applies is
// false (and nothing is launched) otherwise.
int bwd_pair_impl(const void* q, const void* k, const void* v, const void* dout,
                  const float* slopes, float* dk, float* dv, int B, int H, int N, int D, int E,
                  cudaStream_t stream, bool* applies) {
  *applies = false;
  if (D != E) return LA_OK;
  const FwdKernel kern = pick_fwd_kernel(3, true, false);
  int ctas = 0;
  int rc = prepare_fwd_kernel(kern, &ctas);
  if (rc != LA_OK) return rc;
  if (ctas < 2) return LA_OK;
  *applies = true;
  const int nseq = B * H;
  la::fwd::Params p{};
  CUtensorMap m0[4], m1[4];
  int rank0 = 0, rank1 = 0;
  const Strides st = contiguous_strides(H, N, D, E);
  if (!build_maps(v, dout, q, dk, B, H, N, D, E, st, &m0[0], &m0[1], &m0[2], &m0[3], p, &rank0) ||
      !build_maps(k, q, dout, dv, B, H, N, D, E, st, &m1[0], &m1[1], &m1[2], &m1[3], p, &rank1) ||
      rank0 != 3 || rank1 != 3)
    return LA_ERR_CUDA;
  const Plan pl = make_plan(nseq, N, ctas / 2, 0);
  if (pl.total >= (1ll << 31)) return LA_ERR_SHAPE;
  p.out = dk;
  p.out1 = dv;
  for (int j = 0; j < 3; ++j) p.ostride[j] = st.s[3][j];
  p.slopes = slopes;
  p.status = status_word();
  if (!p.status) return LA_ERR_CUDA;
  p.H = H;
  p.N = N;
  apply_plan(pl, nseq, p);
  p.wait_limit_ns = kWaitLimitNs;
  p.tag = launch_tag();
  p.paired = 1;
  void* scratch = nullptr;
  if (pl.bytes) {  // role 0's scratch, then role 1's (pl.bytes is a multiple of 256)
    cudaError_t e = cudaMallocAsync(&scratch, 2 * pl.bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    if (needs_zeroed_ctrl(pl, stream)) {
      e = cudaMemsetAsync(scratch, 0, pl.ctrl, stream);
      if (e == cudaSuccess)
        e = cudaMemsetAsync(static_cast<char*>(scratch) + pl.bytes, 0, pl.ctrl, stream);
      if (e != cudaSuccess) {
        cudaFreeAsync(scratch, stream);
        return cuda_fail(e);
      }
    }
    la::fwd::Params p1{};
    set_scratch(pl, static_cast<char*>(scratch) + pl.bytes, p1);
    set_scratch(pl, scratch, p);
    p.ticket1 = p1.ticket;
    p.flags1 = p1.flags;
    p.prefix1 = p1.prefix;
  }
  rc = launch_fwd(kern, 2 * pl.grid, pl.mode != la::fwd::MODE_TICKETS, stream, m0[0], m0[1],
                  m0[2], m0[3], p, m1);
  if (scratch) {
    const cudaError_t e = cudaFreeAsync(scratch, stream);
    if (e != cudaSuccess && rc == LA_OK) rc = cuda_fail(e);
  }
  return rc;
}

int lightning_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                       const float* slopes, float* dq, float* dk, float* dv, int B, int H, int N,
                       int D, int E, void* stream) {
  if (!q || !k || !v || !dout || !slopes || !dq || !dk || !dv) return LA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned4(slopes))
    return LA_ERR_ALIGN;
  // dq_t = sum_{s<=t} g^(t-s) (dout_t . v_s) k_s: the causal operator on (dout, v, k)
  int rc = fwd_bf16_impl(dout, v, k, slopes, nullptr, nullptr, dq, B, H, N, E, D, 0, stream);
  if (rc != LA_OK) return rc;
  // dk and dv: one paired launch when D == E (the dq launch has checked the
  // shapes, and the pointers are checked above)
  bool paired = false;
  rc = bwd_pair_impl(q, k, v, dout, slopes, dk, dv, B, H, N, D, E,
                     static_cast<cudaStream_t>(stream), &paired);
  if (paired || rc != LA_OK) return rc;
  // dk_s = sum_{t>=s} g^(t-s) (v_s . dout_t) q_t: the anti-causal operator on (v, dout, q)
  rc = fwd_bf16_impl(v, dout, q, slopes, nullptr, nullptr, dk, B, H, N, E, D, 0, stream, nullptr,
                     true);
  if (rc != LA_OK) return rc;
  // dv_s = sum_{t>=s} g^(t-s) (k_s . q_t) dout_t: the anti-causal operator on (k, q, dout)
  return fwd_bf16_impl(k, q, dout, slopes, nullptr, nullptr, dv, B, H, N, D, E, 0, stream, nullptr,
                       true);
}

int lightning_attn_fwd_fused(const void* q, const void* k, const void* v, const void* gate,
                             const float* slopes, const float* norm_weight, float eps, void* out,
                             int B, int H, int N, int D, int E, void* stream) {
  const FusedArgs fa{gate, norm_weight, eps};
  return fwd_bf16_impl(q, k, v, slopes, nullptr, nullptr, out, B, H, N, D, E, 0, stream, nullptr,
                       false, 0, kWaitLimitNs, &fa);
}

int lightning_attn_fwd_fused_ex(const void* q, const void* k, const void* v, const void* gate,
                                const float* slopes, const float* norm_weight, float eps,
                                const float* init_state, float* final_state, void* out, int B,
                                int H, int N, int D, int E, const long long* q_strides,
                                const long long* k_strides, const long long* v_strides,
                                const long long* gate_strides, const long long* out_strides,
                                int chunk, void* stream) {
  const FusedArgs fa{gate, norm_weight, eps};
  const long long* src[5] = {q_strides, k_strides, v_strides, out_strides, gate_strides};
  int given = 0;
  for (const long long* x : src) given += x != nullptr;
  if (given == 0)
    return fwd_bf16_impl(q, k, v, slopes, init_state, final_state, out, B, H, N, D, E, chunk,
                         stream, nullptr, false, 0, kWaitLimitNs, &fa);
  if (given != 5) return LA_ERR_NULL;
  Strides st;
  for (int i = 0; i < 5; ++i)
    for (int j = 0; j < 3; ++j) st.s[i][j] = src[i][j];
  return fwd_bf16_impl(q, k, v, slopes, init_state, final_state, out, B, H, N, D, E, chunk,
                       stream, &st, false, 0, kWaitLimitNs, &fa);
}

int lightning_attn_fault_test_scan_stall(const void* q, const void* k, const void* v,
                                         const float* slopes, float* out, int B, int H, int N,
                                         int chunk, unsigned int wait_limit_ms, void* stream) {
  if (chunk <= 0 || N <= chunk) return LA_ERR_SHAPE;  // needs at least two chunks
  if (wait_limit_ms == 0 || wait_limit_ms > 10000) return LA_ERR_SHAPE;
  return fwd_bf16_impl(q, k, v, slopes, nullptr, nullptr, out, B, H, N, 128, 128, chunk, stream,
                       /*strides=*/nullptr, /*reverse=*/false, /*first_chunk=*/1,
                       1000000ull * wait_limit_ms);
}

int lightning_attn_fwd_noalloc(const void* q, const void* k, const void* v, const float* slopes,
                               float* out, int B, int H, int N, int D, int E, int chunk,
                               void* stream) {
  return fwd_bf16_noalloc_impl(q, k, v, slopes, out, B, H, N, D, E, chunk, stream);
}

int lightning_attn_fwd_f32(const float* q, const float* k, const float* v, const float* slopes,
                           float* out, int B, int H, int N, int D, int E, void* stream) {
  if (!q || !k || !v || !slopes || !out) return LA_ERR_NULL;
  if (!dims_ok(B, H, N, D, E)) return LA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(slopes))
    return LA_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (D == 64 && E == 64) return launch_f32<64, 64>(q, k, v, slopes, out, B, H, N, s);
  if (D == 64 && E == 128) return launch_f32<64, 128>(q, k, v, slopes, out, B, H, N, s);
  if (D == 128 && E == 64) return launch_f32<128, 64>(q, k, v, slopes, out, B, H, N, s);
  if (D == 128 && E == 128) return launch_f32<128, 128>(q, k, v, slopes, out, B, H, N, s);
  return LA_ERR_UNSUPPORTED;
}

int lightning_attn_decode(const void* q, const void* k, const void* v, float* state,
                          const float* slopes, float* out, int B, int H, int D, int E,
                          void* stream) {
  if (!q || !k || !v || !state || !slopes || !out) return LA_ERR_NULL;
  if (!dims_ok(B, H, 1, D, E)) return LA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) ||
      !aligned16(out) || !aligned4(slopes))
    return LA_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (D == 64 && E == 64) return launch_decode<64, 64>(q, k, v, state, slopes, out, B, H, s);
  if (D == 64 && E == 128) return launch_decode<64, 128>(q, k, v, state, slopes, out, B, H, s);
  if (D == 128 && E == 64) return launch_decode<128, 64>(q, k, v, state, slopes, out, B, H, s);
  if (D == 128 && E == 128) return launch_decode<128, 128>(q, k, v, state, slopes, out, B, H, s);
  return LA_ERR_UNSUPPORTED;
}

int lightning_attn_decode_fused(const void* q, const void* k, const void* v, const void* gate,
                                float* state, const float* slopes, const float* norm_weight,
                                float eps, void* out, int B, int H, int D, int E,
                                const long long* q_strides, const long long* k_strides,
                                const long long* v_strides, const long long* gate_strides,
                                const long long* out_strides, void* stream) {
  if (!q || !k || !v || !gate || !state || !slopes || !norm_weight || !out) return LA_ERR_NULL;
  if (!dims_ok(B, H, 1, D, E)) return LA_ERR_SHAPE;
  if (!(eps >= 0.f) || eps > 3.0e38f) return LA_ERR_SHAPE;
  if ((D != 64 && D != 128) || (E != 64 && E != 128)) return LA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(state) ||
      !aligned16(out) || !aligned4(slopes) || !aligned4(norm_weight))
    return LA_ERR_ALIGN;
  const long long* src[5] = {q_strides, k_strides, v_strides, gate_strides, out_strides};
  int given = 0;
  for (const long long* x : src) given += x != nullptr;
  if (given != 0 && given != 5) return LA_ERR_NULL;
  la::DecodeLayerArgs a{};
  long long* dst[5] = {a.qs, a.ks, a.vs, a.gs, a.os};
  const long long width[5] = {D, D, E, E, E};
  for (int i = 0; i < 5; ++i) {
    dst[i][0] = given ? src[i][0] : static_cast<long long>(H) * width[i];
    dst[i][1] = given ? src[i][1] : width[i];
    for (int j = 0; j < 2; ++j)  // 16-byte rows, as every other entry point's tensors
      if (dst[i][j] < 0 || dst[i][j] % 8 != 0 || dst[i][j] >= (1ll << 40)) return LA_ERR_ALIGN;
  }
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.gate = static_cast<const __nv_bfloat16*>(gate);
  a.state = state;
  a.slopes = slopes;
  a.norm_w = norm_weight;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.eps = eps;
  a.H = H;
  const int64_t nbh = static_cast<int64_t>(B) * H;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 64 && E == 64) return launch_decode_layer<64, 64>(a, nbh, st);
  if (D == 64 && E == 128) return launch_decode_layer<64, 128>(a, nbh, st);
  if (D == 128 && E == 64) return launch_decode_layer<128, 64>(a, nbh, st);
  return launch_decode_layer<128, 128>(a, nbh, st);
}

int lightning_attn_state(const void* k, const void* v, const float* slopes,
                         const float* init_state, float* final_state, int B, int H, int N, int D,
                         int E, int chunk, void* stream) {
  return state_impl(k, v, slopes, init_state, final_state, B, H, N, D, E, chunk, stream);
}

int lightning_attn_state_combine(const float* states, int R, const int* chunk_tokens,
                                 const float* slopes, const float* init_state, float* out, int B,
                                 int H, int D, int E, void* stream) {
  if (!slopes || !out || (R > 0 && (!states || !chunk_tokens))) return LA_ERR_NULL;
  if (R < 0 || R > la::COMBINE_MAX_CHUNKS || !dims_ok(B, H, 1, D, E)) return LA_ERR_SHAPE;
  if ((D != 64 && D != 128) || (E != 64 && E != 128)) return LA_ERR_UNSUPPORTED;
  if ((R > 0 && !aligned16(states)) || !aligned16(out) || !aligned4(slopes) ||
      (init_state && !aligned16(init_state)))
    return LA_ERR_ALIGN;
  la::CombineArgs a{};
  for (int j = 0; j < R; ++j) {
    if (chunk_tokens[j] < 0) return LA_ERR_SHAPE;
    a.n[j] = chunk_tokens[j];
  }
  a.states = states;
  a.init = init_state;
  a.slopes = slopes;
  a.out = out;
  a.per_seq4 = static_cast<int64_t>(D) * E / 4;
  a.total4 = static_cast<int64_t>(B) * H * a.per_seq4;
  a.H = H;
  a.R = R;
  const int64_t blocks = (a.total4 + 255) / 256;
  const int64_t cap = 32ll * sm_count();  // grid-stride loop: a few waves of 256 threads
  const int grid = static_cast<int>(blocks < cap ? blocks : cap);
  la::state_combine_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return launch_status();
}

const char* lightning_attn_last_cuda_error(void) { return t_last_cuda_error; }

int lightning_attn_set_cta_limit(int max_ctas, int* previous) {
  if (max_ctas < 0) return LA_ERR_SHAPE;
  const int old = g_cta_limit.exchange(max_ctas);
  if (previous) *previous = old;
  return LA_OK;
}

int lightning_attn_fwd_plan(int B, int H, int N, int chunk, int sms, int* info, int* rec,
                            int max_rec, int* n_rec) {
  if (!info || !n_rec || (max_rec > 0 && !rec)) return LA_ERR_NULL;
  if (!dims_ok(B, H, N, 128, 128) || sms < 1 || chunk < 0 || (chunk % 128) != 0)
    return LA_ERR_SHAPE;
  const int nseq = B * H;
  const Plan pl = make_plan(nseq, N, sms, chunk);
  if (pl.total >= (1ll << 31)) return LA_ERR_SHAPE;
  la::fwd::Params p{};
  p.H = H;
  p.N = N;
  apply_plan(pl, nseq, p);
  info[0] = pl.mode;
  info[1] = pl.grid;
  info[2] = pl.L;
  info[3] = pl.nchunks;
  info[4] = pl.F;
  info[5] = pl.G2;
  info[6] = static_cast<int>(pl.bytes > pl.ctrl ? (pl.bytes - pl.ctrl) / (128 * 128 * sizeof(float)) : 0);
  info[7] = pl.ctrl ? static_cast<int>((pl.ctrl - 8) / 8) : 0;
  p.tag = 1;  // the records show the published flag value of a split as 1
  int n = 0;
  auto put = [&](int cta, int kind, int seq, int a, int b, int flags, int es, int ev, int ps,
                 int pv) {
    if (n < max_rec) {
      int* r = rec + 10 * static_cast<size_t>(n);
      r[0] = cta; r[1] = kind; r[2] = seq; r[3] = a; r[4] = b;
      r[5] = flags; r[6] = es; r[7] = ev; r[8] = ps; r[9] = pv;
    }
    ++n;
  };
  auto put_item = [&](int cta, const la::fwd::Item& it) {
    const int flags = (it.enter ? 1 : 0) | (it.publish ? 2 : 0) | (it.last ? 4 : 0) |
                      (it.phase1 ? 8 : 0);
    put(cta, it.p2 ? 0 : 1, it.seq, it.t0, it.Lc, flags, it.enter_slot,
        static_cast<int>(it.enter_val), it.pub_slot, static_cast<int>(it.pub_val));
  };
  if (pl.mode == la::fwd::MODE_TICKETS) {
    for (int w = 0; w < static_cast<int>(pl.total); ++w) {
      la::fwd::Item it;
      if (!la::fwd::get_item(p, pl.grid, 0, nullptr, w, it)) break;
      put_item(-1, it);
    }
  } else {
    for (int i = 0; i < pl.grid; ++i) {
      uint32_t m[32] = {};
      if (!la::fwd::setup_split(p, pl.grid, i, m)) return LA_ERR_UNSUPPORTED;
      la::fwd::Item it;
      for (int k = 0; la::fwd::get_item(p, pl.grid, i, m, k, it); ++k) {
        put_item(i, it);
        if (it.enter && pl.mode == la::fwd::MODE_SPLIT_SCAN) {
          // the pieces whose local states this entering state chains
          const int64_t lo = static_cast<int64_t>(it.seq) * p.F, hi = lo + it.t0 / 128;
          for (int64_t x = lo; x < hi;) {
            const int64_t y = la::fwd::s1_next(p, pl.grid, x);
            put(i, 2, it.seq, static_cast<int>(x), static_cast<int>(y), 0,
                la::fwd::s1_slot(p, pl.grid, x), 1, 0, 0);
            if (y <= x) return LA_ERR_UNSUPPORTED;
            x = y;
          }
        }
      }
    }
  }
  *n_rec = n;
  return n <= max_rec ? LA_OK : LA_ERR_WORKSPACE;
}

#ifdef LA_TRACE
// Tracing builds only: device buffer of TRACE_CTAS x TRACE_EVENTS x TRACE_SLOTS
// u64 timestamps (or NULL to stop tracing).
int lightning_attn_set_trace(unsigned long long* buf) {
  const cudaError_t e = cudaMemcpyToSymbol(la::fwd::g_trace, &buf, sizeof(buf));
  return e == cudaSuccess ? LA_OK : cuda_fail(e);
}
#endif

const char* lightning_attn_status_string(int status) {
  switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_NULL: return "LA_ERR_NULL: a required pointer is NULL";
    case LA_ERR_SHAPE: return "LA_ERR_SHAPE: invalid sizes";
    case LA_ERR_ALIGN: return "LA_ERR_ALIGN: a tensor pointer is not 16-byte aligned";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: unsupported head geometry";
    case LA_ERR_CUDA: return "LA_ERR_CUDA: a CUDA call or kernel launch failed";
    case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT: a device-side wait ran out of time";
    case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown lightning_attn status";
  }
}

int lightning_attn_device_status(int* status, int reset) {
  if (!status) return LA_ERR_NULL;
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, la::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  *status = v ? LA_ERR_TIMEOUT : LA_OK;
  if (reset) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(la::g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return LA_OK;
}

}  // extern "C"
