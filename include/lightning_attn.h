/*
 * lightning_attn.h -- C ABI of the B200 (sm_100a) Lightning Attention library.
 *
 * The operation (one independent problem per batch row b and head h):
 *
 *     o_t = sum_{s <= t} exp(-lambda_h * (t - s)) * (q_t . k_s) * v_s
 *
 * i.e. causal linear attention with a fixed per-head exponential decay and no
 * normaliser, no softmax and no in-kernel scale.  Sources for the operation:
 *   - "MiniMax-M1" model entry (archdb), field "Configuration of the linear / SSM
 *     layers": Lightning attention with a per-head exponential decay
 *     (ALiBi-style slopes) and a 128x128 state per head.
 *   - same entry, positional-scheme field: Lightning layers use a fixed per-head
 *     decay and no RoPE, so position enters only through the decay.
 *   - "MiniMax-01" (redeep.blog), section "What Makes 1M Context Hard": a
 *     linear-complexity variant that replaces softmax attention.
 *   - Lightning Attention news article (cocoloop), section "El enfoque de
 *     Lightning Attention": complexity reduced from O(n^2) to about O(n).
 * lambda_h is the decay RATE (slope); the per-token factor is gamma_h =
 * exp(-lambda_h), so lambda_h = 0 is plain causal linear attention.  The
 * diagonal s = t is included.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     never frees them and keeps no reference after the call returns.
 *   - Layout is head-major and contiguous: q, k are [B][H][N][D], v is
 *     [B][H][N][E], out is [B][H][N][E] (decode: N is absent).  slopes is a
 *     float32 device array [H].
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream).  They return a status code and never
 *     throw, exit or abort.  Argument errors are detected on the host before any
 *     launch.  A launch failure is reported as LA_ERR_CUDA.
 *   - Preconditions that are NOT checked (checking them would need a device
 *     synchronisation): slopes must be finite and >= 0; out must not alias any
 *     input; decode out must not alias state.
 *   - Device-side waits are bounded in time.  A wait that runs out sets a
 *     sticky per-device status word (read it with lightning_attn_device_status)
 *     and the kernel returns without finishing its outputs.
 */
#ifndef LIGHTNING_ATTN_H_
#define LIGHTNING_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LA_OK = 0,
  LA_ERR_NULL = 1,        /* a required pointer is NULL                         */
  LA_ERR_SHAPE = 2,       /* B, H, N < 1, or sizes overflow 64-bit indexing      */
  LA_ERR_ALIGN = 3,       /* a tensor pointer is not 16-byte aligned            */
  LA_ERR_UNSUPPORTED = 4, /* D or E outside {64, 128} for this entry point      */
  LA_ERR_CUDA = 5,        /* a CUDA runtime/driver call or the launch failed    */
  LA_ERR_TIMEOUT = 6,     /* a bounded device-side wait ran out (see above)     */
  LA_ERR_WORKSPACE = 7    /* caller workspace missing or too small              */
} la_status;

/*
 * Prefill, bf16 inputs, fp32 output ("MiniMax-M1" model entry, linear/SSM
 * layer field: the Lightning layer's causal linear attention with a per-head
 * exponential decay; "MiniMax-01" blog, "What Makes 1M Context Hard": the
 * linear-complexity variant that carries the long context).
 *   q, k : bf16 [B][H][N][D]      v : bf16 [B][H][N][E]
 *   slopes: fp32 [H], lambda_h    out: fp32 [B][H][N][E] (fully overwritten)
 * Zero initial state.  D, E in {64, 128} (the model's geometry is the
 * "128x128 state per head" of the MiniMax-M1 entry, linear-layer field; a
 * 64-wide q/k or v runs on the same 128-wide tiles with the missing columns
 * zero-filled by the tensor maps, which is exact); other D, E return
 * LA_ERR_UNSUPPORTED.  Any N >= 1.
 * Runs on tcgen05 tensor cores (bf16 operands, fp32 accumulation, fp32 state
 * carried on chip).  Work is spread over a persistent grid of one CTA per SM
 * (capped by lightning_attn_set_cta_limit): long sequences are split into
 * parts whose entering states come from a state scan or a hand-over; the
 * scratch (at most 2 states of 64 KiB per CTA, or per (b, h) with an explicit
 * chunk length) is taken with cudaMallocAsync / cudaFreeAsync on `stream`.
 * Where CTAs wait for states other CTAs of the same launch publish (the
 * hand-over when B*H >= CTAs, the split scan when CTAs/8 <= B*H < CTAs), the
 * launch is cooperative: the runtime starts it only with every CTA resident,
 * so a kernel running beside it on another stream (or a share of the SMs
 * held by another process) delays it instead of leaving CTAs waiting for CTAs
 * that cannot start; if the grid can never be resident the call returns
 * LA_ERR_CUDA.  The chunk scan (B*H < CTAs/8, or an explicit chunk) hands
 * work out by ticket in order, so a chunk only waits for a chunk that a
 * running CTA already holds, and needs no such launch.
 */
int lightning_attn_fwd(const void* q, const void* k, const void* v,
                       const float* slopes, float* out,
                       int B, int H, int N, int D, int E, void* stream);

/*
 * lightning_attn_fwd with an optional initial state, an optional final state
 * and an explicit chunk length.
 *   init_state : nullable fp32 [B][H][D][E]; the state before token 0 (zero if
 *                NULL).  Output rows then include exp(-lambda (t+1)) q_t S_0.
 *   final_state: nullable fp32 [B][H][D][E]; receives the state after token
 *                N-1, so a later call (or lightning_attn_decode) can continue
 *                the sequence.
 *   chunk      : tokens per chunk of the parallel sequence split, a multiple
 *                of 128 (LA_ERR_SHAPE otherwise); 0 picks one from B*H, N and
 *                the SM count.  The result does not depend on it beyond
 *                rounding.
 * Same layouts, alignment and errors as lightning_attn_fwd.
 */
int lightning_attn_fwd_ex(const void* q, const void* k, const void* v,
                          const float* slopes, const float* init_state,
                          float* final_state, float* out, int B, int H, int N,
                          int D, int E, int chunk, void* stream);

/*
 * Allocation-free variant of lightning_attn_fwd (the pages have no counterpart:
 * this is an interface for callers, not part of the method).
 *
 * Some callers cannot allocate device memory on the call path: processes whose
 * device memory is carved up once at start-up by their own allocator (which a
 * cudaMallocAsync inside the library would bypass), and latency-critical
 * serving loops where an allocation may block, trim a memory pool or fail under
 * fragmentation.  This entry point performs no allocation and no free.  When a
 * sequence split is used it keeps the chunk-scan scratch in one fixed device
 * array of LA_NOALLOC_SCRATCH_BYTES bytes, compiled into the library; every
 * device that loads the library holds that array until the process exits.
 *
 *   q, k, v, slopes, out, B, H, N, D, E, stream: as lightning_attn_fwd.
 *   chunk: as lightning_attn_fwd_ex (0 = automatic).
 * Scratch needed when the sequences are split: a 256-byte-rounded control
 * block (an 8-byte ticket and one 64-bit flag per state slot) plus 64 KiB per
 * state slot -- 2 B H slots for the chunk scan, at most 2 per SM for the
 * automatic splits.  A call
 * that would need more than LA_NOALLOC_SCRATCH_BYTES returns LA_ERR_WORKSPACE
 * before launching anything.  With chunk = 0 the automatic splits need at most
 * two states per CTA (19.4 MB on a 148-SM B200), within the limit; on a GPU
 * with so many SMs that they would not fit, the call runs whole sequences.
 * The first call on each device loads the library's device code and looks up
 * the array's device address (cudaGetSymbolAddress); make that first call
 * before any stream capture.  The address is looked up again on every call
 * (a host-side table lookup, no allocation), so it stays valid after
 * cudaDeviceReset re-creates the context.  All calls on a device share the
 * one array and it keeps the last
 * call's contents (the chunk scan's counters are cleared with cudaMemsetAsync
 * on `stream` at every call; the other splits' flags carry a value unique to
 * the call): calls whose kernels overlap on the GPU -- e.g. issued on
 * different streams without ordering between them -- race on it and must be
 * serialised by the caller.
 */
#define LA_NOALLOC_SCRATCH_BYTES (20u * 1024u * 1024u)
int lightning_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                               const float* slopes, float* out, int B, int H,
                               int N, int D, int E, int chunk, void* stream);

/*
 * Prefill with caller-chosen strides, otherwise as lightning_attn_fwd_ex
 * (same operation, decays, optional initial/final state and chunk length;
 * bf16 q, k, v, fp32 out, D, E in {64, 128}).  For each of q, k, v and out,
 * {stride_b, stride_h, stride_t} gives the element strides of its batch, head
 * and token dimensions; the innermost dimension (d or e) is contiguous.  This
 * takes the layouts a QKV projection produces without a transposing copy:
 * token-major [B][N][H][D] (strides {N*H*D, D, H*D}) or views into one fused
 * [B][N][3][H][D] buffer (strides {3*N*H*D, D, 3*H*D}, q, k, v H*D elements
 * apart), and token-major outputs [B][N][H][E] (the layout of the layer's
 * output projection input).  The pages show only the per-head computation;
 * the layouts are this library's reading of how a model feeds it.
 * Every stride times the element size (2 bytes for q, k, v; 4 for out) must be
 * a non-negative multiple of 16 bytes below 2^40, and every pointer 16-byte
 * aligned (else LA_ERR_ALIGN); NULL stride arrays give LA_ERR_NULL.  The
 * elements of out must not overlap each other or the inputs (not checked).
 */
int lightning_attn_fwd_strided(const void* q, const void* k, const void* v, const float* slopes,
                               const float* init_state, float* final_state, float* out, int B,
                               int H, int N, int D, int E, const long long* q_strides,
                               const long long* k_strides, const long long* v_strides,
                               const long long* out_strides, int chunk, void* stream);

/*
 * Prefill with fp32 inputs and output: the same operation as
 * lightning_attn_fwd ("MiniMax-M1" model entry, linear/SSM layer field:
 * causal linear attention with a per-head exponential decay), with the same
 * layout and all tensors fp32.  D, E in {64, 128}.  CUDA-core fp32 arithmetic,
 * for callers that need fp32-class accuracy (tensor-core operands would round
 * to bf16).  One CTA per (b, h) sequence, 32-token blocks, the state in shared
 * memory; no scratch.  Errors as lightning_attn_fwd.
 */
int lightning_attn_fwd_f32(const float* q, const float* k, const float* v,
                           const float* slopes, float* out,
                           int B, int H, int N, int D, int E, void* stream);

/*
 * One recurrent decode step for B*H independent (b, h) states: the Lightning
 * layer as a fixed-size recurrent state ("MiniMax-M1" model entry, the count
 * of layers with a fixed-size recurrent state and the linear/SSM layer field's
 * 128x128 state per head), so a generated token costs one read-modify-write
 * of the state whatever the context length.
 *   q, k : bf16 [B][H][D]     v : bf16 [B][H][E]
 *   state: fp32 [B][H][D][E] (row d, column e), read and written IN PLACE
 *   out  : fp32 [B][H][E]
 * Order within the step: state <- exp(-lambda_h) * state + k^T v, then
 * out = q . state (the updated state; consistent with the inclusive diagonal
 * of the prefill).  D, E in {64, 128}.
 */
int lightning_attn_decode(const void* q, const void* k, const void* v,
                          float* state, const float* slopes, float* out,
                          int B, int H, int D, int E, void* stream);

/*
 * Anti-causal prefill: o_t = sum_{s >= t} exp(-lambda_h (s - t)) (q_t . k_s) v_s,
 * the same operation with time reversed (needed by the backward pass below).
 * init_state is the state after the last token (zero if NULL); final_state
 * receives the state at token 0.  Otherwise as lightning_attn_fwd_ex (layouts
 * [B][H][N][*], bf16 q, k, v, fp32 out, D, E in {64, 128}, chunk, errors).
 * The pages state only the causal operator; reversal is the plain reading of
 * what its gradients need.
 */
int lightning_attn_fwd_anticausal(const void* q, const void* k, const void* v, const float* slopes,
                                  const float* init_state, float* final_state, float* out, int B,
                                  int H, int N, int D, int E, int chunk, void* stream);

/*
 * Backward pass of lightning_attn_fwd for training (the abstract: contexts of
 * 1M tokens in training): given dout = dL/d out (bf16 [B][H][N][E]), writes
 * the gradients with respect to the inputs, fp32:
 *   dq_t = sum_{s <= t} g^(t-s) (dout_t . v_s) k_s      dq [B][H][N][D]
 *   dk_s = sum_{t >= s} g^(t-s) (dout_t . v_s) q_t      dk [B][H][N][D]
 *   dv_s = sum_{t >= s} g^(t-s) (q_t . k_s) dout_t      dv [B][H][N][E]
 * (g = exp(-lambda_h); zero initial state; the slopes are not differentiated).
 * dq is the causal operator applied to (dout, v, k); dk and dv are the
 * anti-causal operator applied to (v, dout, q) and (k, q, dout).  With D == E
 * dk and dv share one launch whose CTAs alternate between them on the same
 * work items, so q and dout are streamed from memory about once for both (two
 * launches of the tensor-core kernel on `stream`); otherwise three launches.
 * bf16 inputs as for the forward pass, D, E in {64, 128}; dq, dk, dv 16-byte
 * aligned and not overlapping the inputs or each other (not checked).  Errors
 * as lightning_attn_fwd: LA_ERR_NULL or LA_ERR_ALIGN before any launch, else
 * the first failing launch's code.
 */
int lightning_attn_bwd(const void* q, const void* k, const void* v, const void* dout,
                       const float* slopes, float* dq, float* dk, float* dv, int B, int H, int N,
                       int D, int E, void* stream);

/*
 * The layer around the operator, fused into the prefill kernel ("MiniMax-M1"
 * model entry, linear-layer field: SiLU on Q, K, V, RMSNorm on the output;
 * gate field: a sigmoid gate on the output after the RMSNorm, before the
 * output projection):
 *   y_t = w_h * RMSNorm(o_t) * sigmoid(gate_t),   o = operator(silu(q), silu(k), silu(v))
 *   RMSNorm(o_t) = o_t / sqrt(mean_e(o_te^2) + eps), over each head's E outputs
 * (the pages do not say which axis the RMSNorm covers; this reading is the one
 * a per-head store can compute).
 *   q, k : bf16 [B][H][N][D], the raw projections (SiLU is applied here)
 *   v    : bf16 [B][H][N][E], raw;   gate: bf16 [B][H][N][E], before the sigmoid
 *   norm_weight: fp32 [H][E]   eps: finite, >= 0 (else LA_ERR_SHAPE)
 *   out  : bf16 [B][H][N][E]
 * SiLU is applied in shared memory as the tiles arrive (the MUFU tanh gives the
 * sigmoids), the norm, weight and gate in the epilogue, which stores bf16:
 * 256 B of output per token-head instead of 512.  Zero initial state; D, E in
 * {64, 128}; contiguous tensors, 16-byte aligned (else LA_ERR_ALIGN); errors
 * otherwise as lightning_attn_fwd.  lightning_attn_fwd_fused_ex adds strides
 * and the state in and out.
 */
int lightning_attn_fwd_fused(const void* q, const void* k, const void* v, const void* gate,
                             const float* slopes, const float* norm_weight, float eps, void* out,
                             int B, int H, int N, int D, int E, void* stream);

/*
 * The fused layer (as lightning_attn_fwd_fused) for a model's layer: inputs
 * read in the layouts a QKV projection writes, and the recurrent state handed
 * in and out so a sequence can be prefilled in pieces and then continued token
 * by token with lightning_attn_decode_fused ("MiniMax-M1" model entry:
 * linear-layer field -- SiLU on Q, K, V, RMSNorm on the output, 128x128 state
 * per head; gate field -- sigmoid gate after the RMSNorm; the count of layers
 * with a fixed-size recurrent state).
 *   init_state : nullable fp32 [B][H][D][E], the state before token 0 of the
 *                recurrence on the activated k, v (zero if NULL)
 *   final_state: nullable fp32 [B][H][D][E], receives the state after token N-1
 *   q_strides, k_strides, v_strides, gate_strides, out_strides: {b, h, t}
 *                element strides of each tensor (the last dimension
 *                contiguous), all five NULL for contiguous head-major
 *                [B][H][N][*] tensors, else all five non-NULL (LA_ERR_NULL
 *                otherwise).  E.g. token-major [B][N][H][*] is {N*H*W, W,
 *                H*W}; slices of one fused [B][N][3][H][D] projection output
 *                {3*N*H*D, D, 3*H*D}.  Every stride times 2 bytes a multiple of
 *                16 below 2^40, every pointer 16-byte aligned (LA_ERR_ALIGN).
 *                The elements of out must not overlap each other or the inputs
 *                (not checked).
 *   chunk      : as lightning_attn_fwd_ex.
 * Everything else -- the computation, eps, norm_weight [H][E], bf16 out,
 * D, E in {64, 128}, the errors -- as lightning_attn_fwd_fused.
 */
int lightning_attn_fwd_fused_ex(const void* q, const void* k, const void* v, const void* gate,
                                const float* slopes, const float* norm_weight, float eps,
                                const float* init_state, float* final_state, void* out, int B,
                                int H, int N, int D, int E, const long long* q_strides,
                                const long long* k_strides, const long long* v_strides,
                                const long long* gate_strides, const long long* out_strides,
                                int chunk, void* stream);

/*
 * One decode step of the fused layer: the layer's fixed-size recurrent state
 * advanced by one token ("MiniMax-M1" model entry, the count of layers with a
 * fixed-size recurrent state; linear-layer field: SiLU on Q, K, V, RMSNorm on
 * the output; gate field: sigmoid gate after the RMSNorm), per (b, h):
 *   state <- exp(-lambda_h) state + silu(k)^T silu(v);   o = silu(q) . state
 *   out    = norm_weight[h] * o / sqrt(mean_e(o_e^2) + eps) * sigmoid(gate)
 *   q, k : bf16 [B][H][D], raw projections     v, gate : bf16 [B][H][E], raw
 *   state: fp32 [B][H][D][E], contiguous, updated IN PLACE (the final_state of
 *          lightning_attn_fwd_fused_ex continues here)
 *   norm_weight: fp32 [H][E]   eps: finite, >= 0 (else LA_ERR_SHAPE)
 *   out  : bf16 [B][H][E]
 *   *_strides: {b, h} element strides of q, k, v, gate and out, all five NULL
 *          for the contiguous layouts above, else all five non-NULL; each a
 *          non-negative multiple of 8 elements below 2^40 (LA_ERR_ALIGN).
 * D, E in {64, 128}; every pointer 16-byte aligned except slopes and
 * norm_weight (4).  One CTA per (b, h); HBM-bound like lightning_attn_decode.
 */
int lightning_attn_decode_fused(const void* q, const void* k, const void* v, const void* gate,
                                float* state, const float* slopes, const float* norm_weight,
                                float eps, void* out, int B, int H, int D, int E,
                                const long long* q_strides, const long long* k_strides,
                                const long long* v_strides, const long long* gate_strides,
                                const long long* out_strides, void* stream);

/*
 * The state pass alone: the recurrent state after N tokens,
 *   final_state = exp(-lambda N) S_0 + sum_t exp(-lambda (N-1-t)) k_t^T v_t,
 * without the outputs ("MiniMax-M1" model entry: the linear layers' fixed-size
 * recurrent state, 128x128 per head).  Reads only k and v (512 B per
 * token-head at D = E = 128 instead of the prefill's 1280): for a prompt prefix
 * whose outputs are not needed (the state is what a later prefill or decode
 * continues from), and for the per-chunk states of a sequence split across
 * GPUs (lightning_attn_state_combine).
 *   k : bf16 [B][H][N][D]     v : bf16 [B][H][N][E]    slopes: fp32 [H]
 *   init_state : nullable fp32 [B][H][D][E] (S_0; zero if NULL)
 *   final_state: fp32 [B][H][D][E], fully overwritten (required)
 *   chunk      : as lightning_attn_fwd_ex; 0 picks whole sequences when B*H
 *                fills the grid, else chunks of 1024-8192 tokens chained by
 *                a ticketed scan (scratch from cudaMallocAsync on `stream`)
 * Runs the prefill kernel's local-state pass (tcgen05 K~^T V products into a
 * TMEM state).  D, E in {64, 128}; errors as lightning_attn_fwd.
 */
int lightning_attn_state(const void* k, const void* v, const float* slopes,
                         const float* init_state, float* final_state, int B, int H, int N, int D,
                         int E, int chunk, void* stream);

/*
 * Combines the states of R consecutive chunks of B*H sequences into the state
 * after all of them: with L_j the state of chunk j (n_j tokens) from a zero
 * initial state (lightning_attn_state, init_state NULL),
 *   out = gamma^(n_0 + ... + n_{R-1}) S_0 + sum_j gamma^(n_{j+1} + ... + n_{R-1}) L_j
 * (gamma = exp(-lambda_h); the recurrence is linear in its initial state).
 * This is the one exchange step of a sequence split across GPUs (the
 * abstract's 4M-token inference context): each rank computes L_r of its own
 * chunk, the L_r are all-gathered, and rank r combines L_0 .. L_{r-1} into the
 * entering state of its prefill (lightning_attn_fwd_ex init_state).
 *   states      : fp32 [R][B][H][D][E] (nullable if R = 0), the layout of an
 *                 all-gather of [B][H][D][E] tensors
 *   R           : 0 .. 256 (LA_ERR_SHAPE beyond)
 *   chunk_tokens: HOST array of R token counts (>= 0)
 *   init_state  : nullable fp32 [B][H][D][E] (S_0; zero if NULL)
 *   out         : fp32 [B][H][D][E]; must not overlap the inputs
 * One CUDA-core kernel, HBM-bound (R + 1 states read, one written).
 * D, E in {64, 128}; 16-byte aligned state pointers (LA_ERR_ALIGN).
 */
int lightning_attn_state_combine(const float* states, int R, const int* chunk_tokens,
                                 const float* slopes, const float* init_state, float* out, int B,
                                 int H, int D, int E, void* stream);

/*
 * Fault-injection hook for testing the bounded device-side waits (an interface
 * for tests; the pages have no counterpart).  Runs the chunked bf16 prefill
 * (D = E = 128, chunk a multiple of 128 with N > chunk) but hands out work
 * starting at chunk 1: chunk 0 is never processed, so every chunk-1 item waits
 * on a publication flag that nothing sets.  Each device-side wait of this
 * launch gives up after wait_limit_ms milliseconds (1..10000); the kernel then
 * records LA_ERR_TIMEOUT in the device status word (read it with
 * lightning_attn_device_status), waits for its own copies and MMAs in flight,
 * releases its tensor memory and returns.  `out` is left unspecified.  No
 * fault, trap or unbounded wait is involved; the context stays usable.
 */
int lightning_attn_fault_test_scan_stall(const void* q, const void* k,
                                         const void* v, const float* slopes,
                                         float* out, int B, int H, int N,
                                         int chunk, unsigned int wait_limit_ms,
                                         void* stream);

/*
 * Caps the persistent grid of every later bf16 prefill-kernel launch of this
 * process (lightning_attn_fwd, _ex, _strided, _anticausal, _bwd, _fused,
 * _noalloc) at max_ctas CTAs; 0 removes the cap (one CTA per SM).  For
 * leaving SMs to other work that runs beside the prefill (a decode step on
 * another stream, another process); the work splits are planned for the
 * capped grid, so results do not depend on it beyond rounding.  An interface
 * for callers, with no counterpart on the pages.  *previous (nullable)
 * receives the old cap.  Returns LA_ERR_SHAPE for max_ctas < 0.  The setting
 * is one atomic word shared by all threads; a call that is planning its
 * launch while another thread changes it uses either value.
 */
int lightning_attn_set_cta_limit(int max_ctas, int* previous);

/*
 * Text of the CUDA runtime error behind the calling thread's most recent
 * LA_ERR_CUDA (static string, never NULL; "no error" before any).
 */
const char* lightning_attn_last_cuda_error(void);

/*
 * Scheduling diagnostic (an interface for tests; the pages have no
 * counterpart: how work is spread over the SMs is this implementation's own).
 * Runs on the host only, needs no GPU and touches no device memory.  For a
 * bf16 prefill of B*H sequences of N tokens (D = E = 128) with chunk length
 * `chunk` (0 = automatic) on a GPU with `sms` SMs, reports the plan and every
 * work item the prefill kernel would process:
 *   info[8]: mode (0 whole sequences / chunk scan with tickets, 1 balanced
 *            hand-over, 2 split scan), grid size, chunk length, chunks per
 *            sequence, split-scan first-part blocks F, split-scan output CTAs
 *            over the first parts G2, state slots, 64-bit flags.
 *   rec[10 * i .. 10 * i + 9] for record i: cta (-1 for ticket items), kind
 *            (0 outputs, 1 local state only, 2 a local state chained into the
 *            preceding kind-0 record's entering state), sequence, then for
 *            kinds 0/1 first token and token count, for kind 2 stream blocks
 *            [x, y); flags (1 enters from a published state, 2 publishes its
 *            final state, 4 ends its sequence, 8 computes its local state
 *            first); entering slot and flag value; publishing slot and value (the
 *            chunk scan's values are chunk numbers; a hand-over or split-scan
 *            flag shows 1 here and carries a tag unique to the launch on the
 *            device, so its scratch needs no zeroing).
 * Records are listed per CTA in processing order.  *n_rec receives the
 * number of records; returns LA_ERR_WORKSPACE (records beyond max_rec not
 * written) if max_rec is too small, LA_ERR_SHAPE / LA_ERR_NULL on bad
 * arguments.
 */
int lightning_attn_fwd_plan(int B, int H, int N, int chunk, int sms, int* info, int* rec,
                            int max_rec, int* n_rec);

/* Human-readable name of a la_status value (static string, never NULL). */
const char* lightning_attn_status_string(int status);

/*
 * Reads the calling thread's current device's sticky device-side status word
 * (LA_OK or LA_ERR_TIMEOUT) into *status; if reset != 0 clears it.  This call
 * synchronises with the device.  Returns LA_OK or LA_ERR_NULL / LA_ERR_CUDA.
 * LA_ERR_TIMEOUT covers every device-side abort: a bounded wait that ran out,
 * and (never expected: the host's work split excludes it) a split-scan share
 * whose pieces would not fit the kernel's shared-memory lists.
 */
int lightning_attn_device_status(int* status, int reset);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_ATTN_H_ */
