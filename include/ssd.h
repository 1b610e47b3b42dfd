/*
 * ssd.h -- C ABI of libssd_b200.so, the sm_100a (B200) Mamba-2 SSD hot path.
 *
 * Method: "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching"
 * (arXiv 2603.09555), cited below as [CF-SSD].
 *   - ssd_prefill: the chunked SSD prefill -- per-head scalar decay a = dt*A, its
 *     segment-wise prefix sum exponentiated into the lower-triangular decay matrix, the
 *     intra-chunk dual form (Eq. 3), chunk summary states, the sequential inter-chunk
 *     recurrence, the state-to-output term and the D skip ("Chunked recurrence" and
 *     "Diagonal state matrix" properties).  Its final state initialises the decode cache
 *     (O(1) caching section).
 *   - ssd_decode_step / decode plans: the O(1) cached decode step -- a width-k causal
 *     depthwise conv over k-1 cached inputs, then one recurrence step
 *     h <- exp(dt*A) h + dt * x B^T, y = h C + D x (O(1) caching section), looped on the
 *     device with no host round trip per token ("Compiled on-device loops").
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library never
 *     frees or retains them past the call (a decode plan retains the pointers it was
 *     created with until it is destroyed).  Layouts are row-major (last index
 *     contiguous), densely packed, and every pointer must be 16-byte aligned.
 *   - Scalars per head (dt, A, D), states (h0, h_final, h, conv_state) and conv
 *     parameters are fp32.  x, B, C, y (prefill) and xbc, y (decode) use the io dtype
 *     (SSD_BF16: bfloat16 payloads; SSD_F32: float).
 *   - The library allocates no device memory per call: scratch comes from the caller's
 *     workspace, sized by the matching *_workspace_size query.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; the call returns once it is enqueued.
 *   - Every entry point validates its arguments on the host before launching anything
 *     and returns a status; nothing aborts and nothing throws across the ABI.
 *     ssd_last_error() returns a human-readable detail for the calling thread's last
 *     failure.  Asynchronous CUDA failures surface as SSD_ERR_CUDA on a later call.
 *   - Prefill requires P == 64 and N in {64, 128}; decode requires P == 64 and
 *     N in {64, 128}; any other shape returns SSD_ERR_UNSUPPORTED.
 */
#ifndef SSD_B200_H_
#define SSD_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,  /* null pointer, bad dimension, misalignment, bad enum */
    SSD_ERR_UNSUPPORTED = 2,  /* valid but not implemented shape (e.g. P != 64)     */
    SSD_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed                  */
    SSD_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up                 */
    SSD_ERR_WORKSPACE = 5,    /* workspace pointer null or smaller than required    */
    SSD_ERR_INTERNAL = 6      /* a device-side consistency check failed             */
} ssd_status;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;
typedef enum { SSD_ACT_NONE = 0, SSD_ACT_SILU = 1 } ssd_act;

/* Library version as 10000*major + 100*minor + patch. */
SSD_API int ssd_version(void);

/* Static description of a status code (never NULL). */
SSD_API const char* ssd_status_string(int status);

/* Detail of the calling thread's most recent non-OK status ("" if none). */
SSD_API const char* ssd_last_error(void);

/* ------------------------------------------------------------------------------------
 * Prefill  ([CF-SSD] Eq. 3, "Chunked recurrence", O(1) caching: prefill fills the cache)
 *
 * Shapes: b sequences of T tokens, H heads of head dim P, state size N, G groups of
 * B/C (head h reads group h / (H/G)), chunk length `chunk`.
 *   x       [b][T][H][P]  io dtype      dt [b][T][H] fp32 (positive step sizes, i.e.
 *                                        already passed through softplus)
 *   A       [H] fp32 (negative)         D  [H] fp32
 *   B, C    [b][T][G][N]  io dtype
 *   h0      [b][H][P][N]  fp32, or NULL for a zero initial state
 *   y       [b][T][H][P]  io dtype      (output)
 *   h_final [b][H][P][N]  fp32, or NULL to skip (output; may alias h0 exactly)
 * Computes, per (sequence, head), the result of the recurrence
 *   h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T,  y_t = h_t C_t + D x_t,  h_{-1} = h0
 * through the chunked dual form.  T need not be a multiple of `chunk`: the last chunk
 * is then shorter.  T == 0 or b == 0 is a no-op apart from h_final = h0 (or zeros).
 * chunk must be 64, 128 or 256.  x, B, C, dt, A, D must not alias y or h_final, and the
 * workspace (its required size from its start) must overlap no other buffer.
 * Arithmetic: SSD_BF16 inputs with P == 64 and N == 128 run one fused tensor-core kernel
 * (tcgen05 bf16 contractions, fp32 accumulation, fp32 decay in log space, fp32 running
 * state kept on chip), after a tensor-core state pass when (sequence, head) pairs would
 * leave SMs idle (some or all sequences split into segments whose entering states the
 * fused kernel folds from the state pass's results; see ssd_prefill_segments and
 * ssd_prefill_whole_units).  THAT KERNEL IGNORES `chunk`: it always evaluates the chunked
 * form with 128-token chunks (one tcgen05 tile of rows), whatever chunk length is passed
 * (64, 128 or 256 are accepted and give bitwise the same result).  Every chunk length
 * computes the same function; only the rounding and the operation count differ.  Other
 * bf16 shapes and all SSD_F32 inputs run the three-kernel fp32-FMA path, which uses
 * `chunk` as given, with the prefix sums of dt*A kept in fp64 (no TF32).
 * Determinism: no floating-point atomics; the same call gives bitwise the same y and
 * h_final every time.  A sequence's result can depend on the rest of the batch by rounding
 * only: it is bitwise the same whenever the kernels and segment split chosen for the call
 * are the same (both depend on b * H and, on the fp32 path, on the chunk count).
 * The workspace's first 256 bytes hold a device status word (see ssd_prefill_check).
 * Errors: SSD_ERR_INVALID_ARG (null pointer for a required argument, negative size,
 * H % G != 0, bad chunk or dtype, misaligned pointer, overlapping buffers other than
 * h_final == h0), SSD_ERR_UNSUPPORTED (P, N),
 * SSD_ERR_WORKSPACE (workspace too small or NULL while required), SSD_ERR_CUDA.
 * ---------------------------------------------------------------------------------- */
SSD_API size_t ssd_prefill_workspace_size(int b, int T, int H, int P, int N, int G, int chunk,
                                  int io_dtype);

SSD_API int ssd_prefill(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype,
                const void* x, const float* dt, const float* A, const void* B,
                const void* C, const float* D, const float* h0, void* y, float* h_final,
                void* workspace, size_t workspace_bytes, void* stream);

/* ssd_prefill from the raw time step: the step size is formed inside the kernels where they
 * load it ([CF-SSD]: the elementwise chain ahead of the SSD fused into the kernel; the
 * Mamba-2 block's dt pre-processing), so it never takes a separate pass over memory:
 *   dt[b][t][h] = min(max(softplus(dt_raw[b][t][h] + dt_bias[h]), dt_min), dt_max),
 *   softplus(z) = log(1 + exp(z)), computed in fp32 (z itself above 20).
 *   dt_raw  [b][T][H] fp32      dt_bias [H] fp32, or NULL for no bias
 *   dt_min, dt_max: 0 <= dt_min < dt_max; dt_max may be +infinity (no upper clamp).
 * Everything else, the workspace included, is as for ssd_prefill.
 * Errors: as ssd_prefill, plus SSD_ERR_INVALID_ARG for a clamp range outside the rule above
 * (NaN included) or a misaligned dt_bias. */
SSD_API int ssd_prefill_dt_raw(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype,
                       const void* x, const float* dt_raw, const float* dt_bias, float dt_min,
                       float dt_max, const float* A, const void* B, const void* C, const float* D,
                       const float* h0, void* y, float* h_final, void* workspace,
                       size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Context-parallel prefill: one sequence's tokens split over ranks  ([CF-SSD] "Chunked
 * recurrence": the state entering a stretch of tokens is the decayed sum of the states the
 * earlier stretches leave behind, and y is linear in that state)
 *
 * Rank r holds the consecutive tokens [T_0 + ... + T_{r-1}, ... + T_r) of every sequence.
 *   1. ssd_prefill_local_state: the state its tokens leave when started from zero, and
 *      their total log decay sum(dt * A), per (sequence, head);
 *   2. the caller all-gathers both across ranks, rank-major (one NCCL all-gather each);
 *   3. ssd_prefill_context_scan: the state entering this rank's tokens;
 *   4. ssd_prefill with h0 = that state: this rank's y and the state after its tokens (the
 *      whole sequence's final state on the last rank).
 * The result equals one ssd_prefill over the whole sequence up to rounding.
 * ---------------------------------------------------------------------------------- */

/* Workspace bytes for ssd_prefill_local_state (0 for shapes it does not take or b == 0 or
 * T == 0). */
SSD_API size_t ssd_prefill_local_state_workspace_size(int b, int T, int H, int P, int N, int G,
                                                      int io_dtype);

/* Step 1.  x [b][T][H][P] bf16, dt [b][T][H] fp32 (positive), A [H] fp32, B [b][T][G][N] bf16 as
 * for ssd_prefill; outputs h_local [b][H][P][N] fp32 (the recurrence over these T tokens
 * from h = 0) and log_decay [b][H] fp32 (sum over the tokens of dt * A).  Runs the
 * tensor-core state pass (the tokens cut into pieces to fill the SMs) and a fold of the
 * pieces.  T == 0 writes zeros.  Tensor-core shapes only: bf16, P = 64, N = 128.
 * Errors: SSD_ERR_INVALID_ARG (bad shape or pointer, outputs overlapping inputs or each
 * other, the workspace overlapping any of them), SSD_ERR_UNSUPPORTED (other dtypes or P,
 * N), SSD_ERR_WORKSPACE, SSD_ERR_CUDA. */
SSD_API int ssd_prefill_local_state(int b, int T, int H, int P, int N, int G, int io_dtype,
                                    const void* x, const float* dt, const float* A, const void* B,
                                    float* h_local, float* log_decay, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Step 3.  h_local_all [world][b][H][P][N] and log_decay_all [world][b][H] (fp32, as
 * all-gathered, rank-major); h0 [b][H][P][N] the state before the first rank's tokens (NULL:
 * zeros).  Writes h_in [b][H][P][N] = the state entering rank `rank`'s tokens:
 *   run = h0; for q < rank: run = exp(log_decay_all[q]) * run + h_local_all[q].
 * Only ranks q < rank are read (may be NULL for rank 0).  h_in may alias h0 exactly.
 * Errors: SSD_ERR_INVALID_ARG (rank outside [0, world), b < 0, H < 1, bad pointers or
 * overlaps), SSD_ERR_UNSUPPORTED (P != 64 or N != 128), SSD_ERR_CUDA. */
SSD_API int ssd_prefill_context_scan(int world, int rank, int b, int H, int P, int N,
                                     const float* h0, const float* h_local_all,
                                     const float* log_decay_all, float* h_in, void* stream);

/* Synchronises `stream` and returns the device-side status recorded by the most recent
 * ssd_prefill that used `workspace` (SSD_OK, or SSD_ERR_TIMEOUT if a bounded wait inside
 * the tensor-core kernel expired, or SSD_ERR_INTERNAL for a failed device consistency
 * check: a dynamic shared-memory base that is not 1024-byte aligned, or a tensor-memory
 * allocation whose address never reached the CTA), then clears it; ssd_last_error names
 * the wait site or the check.  Each ssd_prefill call resets the status word first. */
SSD_API int ssd_prefill_check(void* workspace, void* stream);

/* Failure-detection test hook.  Arms a one-shot fault for the next ssd_prefill in this
 * process that takes the tensor-core path (bf16, P = 64, N = 128): its TMA producer issues
 * no loads, so every consumer's bounded wait runs out after `wait_limit_ns` (instead of the
 * default 2 s), the kernel records SSD_ERR_TIMEOUT with the site of the first expired wait,
 * drains, frees its tensor memory and exits; ssd_prefill_check then returns
 * SSD_ERR_TIMEOUT and the CUDA context stays usable.  The y and h_final of that call are
 * undefined.  Nothing faults, traps or spins without a limit.
 * Errors: SSD_ERR_INVALID_ARG if wait_limit_ns is outside [1e6, 1e10] (1 ms .. 10 s). */
SSD_API int ssd_debug_starve_next_prefill(unsigned long long wait_limit_ns);

/* Test hook for the sequence split of the tensor-core prefill.  With nseg >= 1, every
 * following tensor-core ssd_prefill (and ssd_prefill_workspace_size) in this process
 * splits each sequence into min(nseg, ceil(T / 128)) segments of whole 128-token blocks
 * instead of the count its cost model picks; nseg = 0 restores the cost model.  The
 * result is the same function either way (only rounding differs): segments after the
 * first start from the fold of the earlier segments' local end states.
 * Not thread-safe against concurrent prefill calls.
 * Errors: SSD_ERR_INVALID_ARG if nseg < 0. */
SSD_API int ssd_debug_force_prefill_segments(int nseg);

/* The same hook with the whole-unit count too: the first n_full (sequence, head) units (in
 * order b * H + h) run in one pass and every later unit is split into nseg segments (the
 * cost model's "ragged last wave" split).  n_full is clamped to b * H; nseg = 0 restores
 * the cost model.  Errors: SSD_ERR_INVALID_ARG if n_full < 0 or nseg < 0. */
SSD_API int ssd_debug_force_prefill_split(int n_full, int nseg);

/* Test and measurement hook: with on = 1, every following ssd_prefill / ssd_prefill_dt_raw
 * in this process (and ssd_prefill_workspace_size, ssd_prefill_segments,
 * ssd_prefill_whole_units) takes the fp32-FMA path even for shapes the tensor-core kernel
 * takes.  That path evaluates the chunked dual form with chunks of exactly `chunk` tokens,
 * so it serves the literal chunk-length sweep ([CF-SSD] "Chunked recurrence": the chunk
 * size trades arithmetic intensity against sequential overhead) at any shape; it is an
 * order of magnitude slower than the tensor-core kernel.  on = 0 restores the default.
 * Not thread-safe against concurrent prefill calls.
 * Errors: SSD_ERR_INVALID_ARG if on is not 0 or 1. */
SSD_API int ssd_debug_force_fma_prefill(int on);

/* Decay-precision ablation for the tensor-core prefill ([CF-SSD] "Precision management":
 * decay parameters held in log space in fp32 and exponentiated at compute time; bf16 for
 * the decay exponentiation alone shifts the output).  mode 0 (the default) keeps every
 * decay quantity in fp32; mode 1 rounds every exponentiated decay factor to bf16; mode 2
 * rounds the log-space prefix sums of dt*A to bf16 before they are exponentiated.  Applies
 * to every following tensor-core ssd_prefill in this process until reset with 0.  For
 * measuring the effect only: modes 1 and 2 are less accurate by design.
 * Errors: SSD_ERR_INVALID_ARG if mode is not 0, 1 or 2. */
SSD_API int ssd_debug_decay_precision(int mode);

/* Segments per sequence that ssd_prefill would use for this shape: 1 when the whole
 * sequence runs in one pass (every shape outside the tensor-core path, and tensor-core
 * shapes whose sequence-heads fill the SMs of the current device in whole waves), else the
 * count of 128-token-aligned segments of each split sequence-head (see ssd_prefill: local
 * end states, then the fused pass per segment, which folds the earlier segments' states).
 * Returns 0 for an invalid shape.  Host-only; nothing is enqueued. */
SSD_API int ssd_prefill_segments(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype);

/* How many (sequence, head) pairs ssd_prefill runs whole, in one pass each, for this
 * shape: b*H when nothing is split, 0 when every pair is split into
 * ssd_prefill_segments(...) segments, or the pairs of the whole waves of CTAs when only the
 * pairs of a ragged last wave are split (pairs are ordered bi * H + head).  Returns -1 for
 * an invalid shape.  Host-only; nothing is enqueued. */
SSD_API int ssd_prefill_whole_units(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype);

/* ------------------------------------------------------------------------------------
 * Cached decode step  ([CF-SSD] O(1) caching section)
 *
 * One token for every (layer, sequence) pair, all layers in one launch.  With
 * Dc = H*P + 2*G*N conv channels ordered [x (H*P) | B (G*N) | C (G*N)]:
 *   h          [layers][b][H][P][N]   fp32, updated IN PLACE
 *   conv_state [layers][b][Dc][k-1]   fp32, updated IN PLACE (oldest input first)
 *   xbc        [layers][b][Dc]        io dtype: this token's pre-conv inputs
 *   dt         [layers][b][H]         fp32 (positive)
 *   A, D       [layers][H]            fp32
 *   conv_w     [layers][Dc][k]        fp32: tap i multiplies window[i], where window =
 *                                     [conv_state[..][0..k-2], xbc] (tap k-1 = current)
 *   conv_b     [layers][Dc]           fp32
 *   y          [layers][b][H][P]      io dtype (output)
 * Per pair: u = act(conv(window) + bias); conv_state <- window[1..k-1];
 * x, Bv, Cv = split(u); per head: h = exp(dt*A) h + dt * x Bv^T; y = h Cv + D x.
 * act is SSD_ACT_NONE or SSD_ACT_SILU; kconv must be 4.  The workspace (see
 * ssd_decode_workspace_size) holds per-(layer, sequence, group) arrival counters that
 * the call zero-fills itself; calls sharing one workspace must be stream-ordered.  The
 * buffers the step writes (h, conv_state, y, the workspace) must overlap neither one another
 * nor any input; inputs may share memory with one another.
 * Errors: as for ssd_prefill (SSD_ERR_INVALID_ARG for an overlap named above).
 * ---------------------------------------------------------------------------------- */
SSD_API size_t ssd_decode_workspace_size(int layers, int b, int G);

SSD_API int ssd_decode_step(int layers, int b, int H, int P, int N, int G, int kconv, int act,
                    int io_dtype, float* h, float* conv_state, const void* xbc,
                    const float* dt, const float* A, const float* D, const float* conv_w,
                    const float* conv_b, void* y, void* workspace, size_t workspace_bytes,
                    void* stream);

/* ------------------------------------------------------------------------------------
 * Allocation-free decode step  (the paper has no counterpart: this is an integration
 * entry point, not part of the method)
 *
 * For callers that cannot allocate device memory or hand the library a workspace: code
 * that runs inside an engine's enqueue/plugin hook where the engine owns every byte of
 * device memory, code recorded while a CUDA graph is being captured (cudaMalloc is not
 * allowed then), and real-time serving loops that forbid allocation after start-up.
 * Same arguments, semantics and errors as ssd_decode_step, without the workspace.  The
 * scratch it needs (one 32-bit arrival counter per (layer, sequence, group)) lives in a
 * file-scope device array of SSD_DECODE_NOALLOC_MAX_COUNTERS counters (256 KiB) that
 * every GPU which loads the library keeps until the process exits; layers*b*G above
 * that limit returns SSD_ERR_INVALID_ARG.  The first call in a CUDA context looks up the
 * array's device address with that context current (cudaGetSymbolAddress) and caches it
 * under the context's unique id, so make that first call before any stream capture; a
 * context created later on the same device (after cudaDeviceReset, or a caller's own
 * context) is looked up afresh, never served an address from a context that is gone.  Each call clears the counters it uses
 * (cudaMemsetAsync on `stream`) and calls no cudaMalloc, cudaFree or allocating
 * routine.  All calls on a device share the one array: calls that overlap on the GPU
 * (unordered streams) race on it and corrupt each other's conv windows.
 * ---------------------------------------------------------------------------------- */
#define SSD_DECODE_NOALLOC_MAX_COUNTERS 65536

SSD_API int ssd_decode_step_noalloc(int layers, int b, int H, int P, int N, int G, int kconv,
                                    int act, int io_dtype, float* h, float* conv_state,
                                    const void* xbc, const float* dt, const float* A,
                                    const float* D, const float* conv_w, const float* conv_b,
                                    void* y, void* stream);

/* ------------------------------------------------------------------------------------
 * On-device decode loop  ([CF-SSD] "Compiled on-device loops")
 *
 * A plan records n_steps decode steps as one CUDA graph (a counter reset, then n_steps
 * dependent step kernels) so that a launch runs every step with no host involvement.
 * Step t of a launch (t = 0 .. n_steps-1, restarting at 0 on every launch) reads
 * xbc_ring[t % ring] ([ring][layers][b][Dc]) and
 * dt_ring[t % ring] ([ring][layers][b][H]) and writes y_ring[t % ring]
 * ([ring][layers][b][H][P]); h and conv_state are carried in place from step to step.
 * The plan keeps every pointer it was given; the caller keeps them alive and unmoved
 * until ssd_decode_plan_destroy.  A plan may be launched any number of times (each
 * launch continues from the current h / conv_state).  Plans are not thread-safe.
 * ---------------------------------------------------------------------------------- */
typedef struct ssd_decode_plan ssd_decode_plan;

SSD_API int ssd_decode_plan_create(ssd_decode_plan** plan, int layers, int b, int H, int P, int N,
                           int G, int kconv, int act, int io_dtype, float* h,
                           float* conv_state, const void* xbc_ring, const float* dt_ring,
                           int ring, const float* A, const float* D, const float* conv_w,
                           const float* conv_b, void* y_ring, int n_steps, void* workspace,
                           size_t workspace_bytes);

SSD_API int ssd_decode_plan_launch(ssd_decode_plan* plan, void* stream);

SSD_API int ssd_decode_plan_destroy(ssd_decode_plan* plan);

/* n_steps decode steps as one graph launch on `stream`, with no host synchronisation inside:
 * a plan as above is built, launched once and destroyed (the graph is freed by the driver
 * when the launch completes).  Same arguments, layouts and errors as ssd_decode_plan_create
 * plus the stream; every pointer, the workspace included, must stay valid until the
 * launch has completed.  For repeated loops over the same buffers, keep a plan instead:
 * building the graph costs host time per call. */
SSD_API int ssd_decode_loop(int layers, int b, int H, int P, int N, int G, int kconv, int act, int io_dtype,
                            float* h, float* conv_state, const void* xbc_ring, const float* dt_ring, int ring,
                            const float* A, const float* D, const float* conv_w, const float* conv_b,
                            void* y_ring, int n_steps, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Measurement hooks (no counterpart on the pages; used by the benchmark)
 *
 * ssd_launch_count: total number of kernels this library has enqueued in this process
 * (a decode plan launch counts its n_steps step kernels; memsets are not counted).
 * ssd_profile_begin: from now on, every kernel launch is bracketed by a pair of CUDA
 * events recorded on the launching stream (at most 65536 launches are kept).
 * ssd_profile_end: waits for the recorded events, stops recording and reports per
 * kernel name the number of launches and the summed event time in milliseconds, in
 * first-launch order.  Returns the number of entries written (<= max_entries) or a
 * negative ssd_status on failure.  Not thread-safe; kernels inside a decode plan are
 * not bracketed (the plan launch as a whole is, under the name "decode_plan").
 * ---------------------------------------------------------------------------------- */
typedef struct {
    char name[48];
    int launches;
    double total_ms;
} ssd_kernel_time;

SSD_API uint64_t ssd_launch_count(void);
SSD_API int ssd_profile_begin(void);
SSD_API int ssd_profile_end(ssd_kernel_time* out, int max_entries);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_H_ */
