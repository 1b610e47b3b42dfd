// prefill_tc.cu -- chunked SSD prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA),
// one fused kernel for bf16 inputs with P = 64, N = 128.
//
// Method: "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching"
// (arXiv 2603.09555).  Inside a block of tokens the recurrence is evaluated in its dual
// form (Eq. 3): scores = (C B^T) o L with L[i][j] = exp(cs_i - cs_j) dt_j for j <= i (a
// fixed causal mask, "Static control flow"), y_intra = scores X; the block's summary
// state B^T (w o X) with w_j = exp(cs_last - cs_j) dt_j; the state entering the block
// reaches token i as exp(cs_i) C_i . H; and a sequential recurrence carries the state
// from block to block ("Chunked recurrence").  The D skip is folded into the diagonal of
// the score matrix (j = i contributes D x_i).
//
// Design (B200): one CTA walks one (sequence, head) through its 128-token blocks (128 =
// the M of one tcgen05 MMA), so x, B and C are read from HBM once, y is written once and
// the fp32 running state never leaves the chip.  A chunk of L = 256 tokens is processed
// as two such blocks with the state handed between them -- the same dual form over a
// shorter segment, identical in exact arithmetic.
//
// Only the state recurrence is sequential; the dual form of a block needs nothing from the
// blocks before it.  The kernel therefore runs two pipelines that meet only at the output:
// the scores path (C B^T -> P -> P X) runs up to a block ahead of the state path
// (w o X -> S -> H -> C H^T), each with its own MMA-issuing warp, and every TMEM buffer the
// scores path needs is doubled so it never waits for the block before.
//
//   warp 0       TMA producer: C and B (two 64-column 128B-swizzled boxes each) into a
//                2-slot ring, X into a 3-slot ring
//   warp 1       TMEM owner; issues the scores path (one elected lane):
//                  CB(k)     = C B^T          (M=128 i, N=128 j, K=128 n)  SS -> CB/P buffer k&1
//                  Y(k)      = P(k) X(k)      (M=128 i, N=64 p,  K=128 j)  TS, P in buffer k&1
//                in the order CB(k+1), Y(k), so C B^T runs one block ahead
//   warp 2       issues the state path:
//                  S(k)^T    = B^T (w o X)    (M=128 n, N=64 p,  K=128 j)  SS
//                  Yst(k)    = C H(k)^T       (M=128 i, N=64 p,  K=128 n)  SS -> buffer k&1
//   warps 3-10   "scores" group (2 warps per TMEM lane quadrant): P = bf16(CB o L) written
//                back IN PLACE over the C B^T columns it was computed from (chunk c of 32
//                score columns -> the first 16 of its 32 columns, bf16 pairs), the A
//                operand of P X; then for the previous block y = Y + exp(cs_i) Yst into a
//                swizzled shared tile (the block's X slot, dead by then)
//   warps 11-18  "state" group (2 warps per quadrant): w o X into shared memory, H <-
//                exp(cs_last) H + S in fp32 registers, its bf16 copy H^T for C H^T
//   warp 19      y store: one TMA tensor store per block, then the X slot goes back to
//                the producer
//   warp 20      "prep": prefix sums of dt*A and every per-token decay term of a block (the
//                scores group's and the state group's), two blocks ahead of their use
//
// A warp whose TMEM lane quadrant is q is warp q (mod 4): warps 3-10 and 11-18 map onto
// the quadrants 3, 0, 1, 2, 3, 0, 1, 2.
//
// Decay arithmetic.  Below the 32x32 diagonal sub-blocks the decay factorises exactly
// as exp(cs_i - cs_e) * exp(cs_e - cs_j) with e the last token of j's 32-token group
// (both factors <= 1: no overflow, underflow only where the true value underflows), so
// those elements cost two multiplies; only the diagonal sub-blocks take one ex2 each.
//
// Every mbarrier wait is bounded by a wall-clock limit; on expiry the kernel records
// SSD_ERR_TIMEOUT in the status word, each group stops at a point all its threads reach
// together, in-flight copies and MMAs are drained, the TMEM is released and the kernel
// returns (no trap, no endless loop).
#include <algorithm>
#include <atomic>
#include <cmath>
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace ssd {
namespace {

constexpr int kBlk = 128;    // tokens per block = MMA M
constexpr int kP = 64;       // head dim
constexpr int kN = 128;      // state size
constexpr int kGroupThreads = 256;  // threads per epilogue group
constexpr int kWarpScores = 3, kWarpState = 11;
constexpr int kWarpStore = kWarpState + 8;         // the y-store warp
constexpr int kWarpPrep = kWarpStore + 1;          // the decay-term warp
constexpr int kThreads = 32 * (kWarpPrep + 1);     // 21 warps
constexpr float kLog2e = 1.4426950408889634f;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t kRegion = kBlk * 128;             // one [128 rows][64 bf16] swizzled box: 16 KB
constexpr uint32_t kCBSlot = 4 * kRegion;            // C (2 regions: n 0..63, 64..127) then B (2)
constexpr uint32_t kSlotC = 0;
constexpr uint32_t kSlotB = 2 * kRegion;
constexpr uint32_t kXRing = 2 * kCBSlot;             // 3 X slots of one region; slot k % 3 holds
                                                     // X(k), then the bf16 y tile of block k
constexpr uint32_t kXs = kXRing + 3 * kRegion;       // w o X
constexpr uint32_t kSH = kXs + kRegion;              // bf16 H^T [n][p]
constexpr uint32_t kSmall = kSH + kRegion;           // barriers and per-token scalars
constexpr uint32_t kSmallBytes = 5120;
constexpr uint32_t kSmemBytes = kSmall + kSmallBytes;
static_assert(kSmemBytes <= 232448 - 1024, "shared memory budget (1 KB of static shared memory beside it)");

// TMEM columns (512 x 128 lanes x 32 bit)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColCBP = 0;     // two 128-column buffers: fp32 C B^T, then bf16 P in place
constexpr uint32_t kColY = 256;     // fp32 Y (64 columns)
constexpr uint32_t kColYst = 320;   // two 64-column C H^T buffers
constexpr uint32_t kColS = 448;     // fp32 S^T (64 columns)
static_assert(kColS + 64 == kTmemCols, "TMEM map");

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

// barrier indices in the small area; [n] = n barriers indexed by block (k & 1, or k % 3)
enum {
    BAR_FULLCB = 0,    // [2] C,B landed (TMA transaction bytes)
    BAR_EMPTYCB = 2,   // [2] C,B slot free: C B^T (issuer 1) and S, C H^T (issuer 2) done  (2 arrivals)
    BAR_FULLX = 4,     // [3] X landed
    BAR_EMPTYX = 7,    // [3] X slot free: its y tile has been read out by the TMA store
    BAR_CBFULL = 10,   // [2] C B^T accumulated in CB/P buffer k & 1
    BAR_PREADY = 12,   // [2] scores group wrote P over it                              (256)
    BAR_PXDONE = 14,   // [2] Y = P X accumulated: the CB/P buffer is free again
    BAR_YFREE = 16,    // scores group read Y                                            (256)
    BAR_PREP = 17,     // [2] the prep warp published a block's decay terms              (1)
    BAR_XSREADY = 19,  // state group wrote w o X                                        (256)
    BAR_SDONE = 20,    // S^T accumulated (w o X read)
    BAR_SFREE = 21,    // state group read S^T                                           (256)
    BAR_HREADY = 22,   // state group wrote bf16 H^T                                     (256)
    BAR_YSTDONE = 23,  // [2] C H^T accumulated (H^T read)
    BAR_YSTFREE = 25,  // [2] scores group read C H^T                                    (256)
    BAR_YSTAGED = 27,  // [3] scores group wrote block k's y tile into X slot k % 3          (256)
    BAR_ARRFREE = 30,  // [2] a block's decay terms read: scores and state warps      (16 warps)
    BAR_DONE1 = 32,    // every MMA of issuer 1 complete (teardown)
    BAR_DONE2 = 33,    // every MMA of issuer 2 complete (teardown)
    BAR_COUNT
};
static_assert(BAR_COUNT * 8 <= 512, "barriers fit ahead of the per-token arrays");
__host__ __device__ constexpr uint32_t bar_count(int i) {
    return (i == BAR_EMPTYCB || i == BAR_EMPTYCB + 1) ? 2u
           : (i == BAR_ARRFREE || i == BAR_ARRFREE + 1) ? 16u
           : (i == BAR_PREADY || i == BAR_PREADY + 1 || i == BAR_YFREE ||
              i == BAR_XSREADY || i == BAR_SFREE || i == BAR_HREADY || i == BAR_YSTFREE || i == BAR_YSTFREE + 1 ||
              (i >= BAR_YSTAGED && i < BAR_YSTAGED + 3))
               ? (uint32_t)kGroupThreads
               : 1u;
}

struct TcParams {
    CUtensorMap tm_x;
    CUtensorMap tm_B;
    CUtensorMap tm_C;
    CUtensorMap tm_y;
    const float* dt;
    DtMap dtm;                   // dt as given, or the softplus pre-processing of raw dt
    const float* A;
    const float* D;
    const float* h0;
    const float* h0_split;       // h0 as read by the first segment of a split unit: h0 itself, or
                                 // a copy when h0 and hf are one buffer (the unit's last segment
                                 // writes hf while its first may not have started)
    float* hf;
    __nv_bfloat16* y;
    int* status;
    int T, H, G;
    // Work split.  A unit is one (sequence, head), u = bi * H + hd.  Units [0, n_full) run
    // whole; each later unit ("split unit" su = u - n_full) is cut into nseg segments of
    // tseg tokens (a multiple of kBlk; the last may be shorter).  The fused kernel's CTAs
    // walk n_full whole units, then the split units' segments in order.
    int n_full, tseg, nseg;
    float* seg_state;            // [su][nseg-1][P][N] fp32: the end state of segment q started
                                 // from zero, except segment 0, which starts from h0; with
                                 // seg_prefix, the prefix pass has turned each into the state
                                 // entering segment q + 1
    float* seg_logdecay;         // [su][nseg-1]: sum of dt*A over a segment
    int seg_prefix;
    unsigned long long wait_ns;  // limit of every bounded wait
    int starve;                  // failure-detection test: the producer issues no loads
};

// per-CTA copy of the wait limit, set before the first wait
__shared__ unsigned long long s_wait_ns;

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait that lets the hardware suspend the thread (up to ~1 ms) until the phase
// completes, instead of spinning on the issue slots other warps need.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
// Programmatic dependent launch.  A grid launched with programmatic stream serialization
// may start while the grid before it in the stream is still running: griddep_wait() blocks
// until that grid has completed and its writes are visible, and griddep_launch() lets the
// next grid in the stream start before this one ends.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Records a failure in the status word (the first one wins).  The word is cleared by the
// grid that runs ahead of every prefill, so the write waits until that grid is done.
__device__ __noinline__ void report_status(int* status, int code) {
    griddep_wait();
    atomicCAS(status, 0, code);
}

// Bounded wait for the phase with `parity` to complete.  Returns false (and makes every
// other role give up) if the CTA is aborting or the limit expires.  The first test is
// inline; the waiting loop is one out-of-line copy shared by every call site, which keeps
// the kernel's hot code small (instruction fetch, not arithmetic, bounds the busy warps).
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                            int where) {
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_sleep(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > s_wait_ns) {
            *abort_flag = 1;
            report_status(status, SSD_ERR_TIMEOUT | (where << 8));
            return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          int where) {
    if (mbar_try(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, abort_flag, status, where);
}
// The same, voted across the warp so that warp-collective tcgen05 instructions after it
// are executed by all lanes or by none.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          int where) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, where));
}
// Drain: bounded wait that never sets the abort flag (used on the way out).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_try(bar, parity) && globaltimer() - t0 < s_wait_ns) {
    }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
// y tile: shared -> global through the async proxy (rows past T are clipped by the map)
__device__ __forceinline__ void tma_store_4d(uint32_t src, const CUtensorMap* tm, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(tm)), "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// TMEM allocation for the whole CTA; returns the allocation's address (the same in every
// thread).  tcgen05.alloc writes the address into a shared-memory slot, which the fence /
// barrier / fence sequence orders before the read.  As a guard on top of that, the slot
// first holds a sentinel (written before the allocation, ordered by a barrier) and every
// thread re-reads it until the address has replaced it (bounded), so no thread can act on
// whatever that shared memory held before the allocation; a diagnostic build that counted
// first reads of the sentinel saw none.  An address that never arrives leaves the sentinel,
// which the caller treats as a failed CTA (status SSD_ERR_INTERNAL).
constexpr uint32_t kTmemSentinel = 0xFFFFFFFFu;
__device__ __forceinline__ uint32_t tmem_alloc_cta(uint32_t* s_tmem, uint32_t cols, bool alloc_warp) {
    volatile uint32_t* slot = s_tmem;
    if (threadIdx.x == 0) *slot = kTmemSentinel;
    __syncwarp();
    __syncthreads();
    if (alloc_warp) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t t = *slot;
    if (t == kTmemSentinel) {
        const unsigned long long t0 = globaltimer();
        while (t == kTmemSentinel && globaltimer() - t0 < kWaitLimitNs) t = *slot;
    }
    return t;
}
__device__ __forceinline__ void group_bar(int id) {
    __syncwarp();  // bar.sync is .aligned: each warp arrives converged
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kGroupThreads) : "memory");
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Decay-precision ablation, a compile-time kernel parameter (kDecay): 0 keeps every decay
// quantity in fp32 (the product); 1 rounds every exponentiated decay factor to bf16; 2
// rounds the log-space prefix sums of dt*A to bf16 before they are exponentiated.
__device__ __forceinline__ float bf16r(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }
template <int kDecay> __device__ __forceinline__ float dlog(float v) { return kDecay == 2 ? bf16r(v) : v; }
template <int kDecay> __device__ __forceinline__ float dexp(float v) { return kDecay == 1 ? bf16r(v) : v; }

// UMMA shared-memory matrix descriptor: 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Whole-warp variants: every lane runs the issuing code (so its operands stay warp-uniform)
// and one elected lane executes the instruction.
__device__ __forceinline__ void mma_ss_w(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_ts_w(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        ::"r"(tmem_d), "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(bar)
        : "memory");
}
// TMEM <-> register moves.  tcgen05.ld/st/wait are .sync.aligned: the whole warp must
// execute them converged, so each macro first reconverges the warp (a store by a few
// lanes or a lane-dependent select ahead of a move may otherwise leave it split).
// tcgen05.ld writes its destination registers, and tcgen05.st
// reads its source registers, asynchronously until the matching tcgen05.wait; each macro
// issues the moves and the wait in ONE asm statement, so the compiler never sees the
// registers as defined (or free) before the wait and cannot reuse, spill or read them
// while the move is still in flight.  The two-load forms take the second address as an
// immediate offset from the first and form it in a register of their own before the first
// load issues: an output of the first load, written asynchronously, can then never be the
// register the second load reads its address from.
#define SSD_TMEM_LD32_WAIT(taddr, r) \
    do { \
    __syncwarp(); \
    asm volatile( \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t" \
        "tcgen05.wait::ld.sync.aligned;" \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), \
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), \
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), \
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), \
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31]) \
        : "r"(taddr) \
        : "memory"); \
    } while (0)
#define SSD_TMEM_LD32x2_WAIT(ta, off, ra, rb) \
    do { \
    __syncwarp(); \
    asm volatile( \
        "{\n\t.reg .b32 tb;\n\tadd.u32 tb, %64, %65;\n\t" \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t" \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [tb];\n\t" \
        "tcgen05.wait::ld.sync.aligned;\n\t}" \
        : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), \
          "=r"(ra[7]), "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), \
          "=r"(ra[14]), "=r"(ra[15]), "=r"(ra[16]), "=r"(ra[17]), "=r"(ra[18]), "=r"(ra[19]), "=r"(ra[20]), \
          "=r"(ra[21]), "=r"(ra[22]), "=r"(ra[23]), "=r"(ra[24]), "=r"(ra[25]), "=r"(ra[26]), "=r"(ra[27]), \
          "=r"(ra[28]), "=r"(ra[29]), "=r"(ra[30]), "=r"(ra[31]), "=r"(rb[0]), "=r"(rb[1]), "=r"(rb[2]), \
          "=r"(rb[3]), "=r"(rb[4]), "=r"(rb[5]), "=r"(rb[6]), "=r"(rb[7]), "=r"(rb[8]), "=r"(rb[9]), \
          "=r"(rb[10]), "=r"(rb[11]), "=r"(rb[12]), "=r"(rb[13]), "=r"(rb[14]), "=r"(rb[15]), "=r"(rb[16]), \
          "=r"(rb[17]), "=r"(rb[18]), "=r"(rb[19]), "=r"(rb[20]), "=r"(rb[21]), "=r"(rb[22]), "=r"(rb[23]), \
          "=r"(rb[24]), "=r"(rb[25]), "=r"(rb[26]), "=r"(rb[27]), "=r"(rb[28]), "=r"(rb[29]), "=r"(rb[30]), \
          "=r"(rb[31]) \
        : "r"(ta), "n"(off) \
        : "memory"); \
    } while (0)
#define SSD_TMEM_LD16x2_WAIT(ta, off, ra, rb) SSD_TMEM_LD16x2_WAIT_(ta, off, ra, rb, "n")
#define SSD_TMEM_LD16x2_WAIT_R(ta, off, ra, rb) SSD_TMEM_LD16x2_WAIT_(ta, off, ra, rb, "r")
#define SSD_TMEM_LD16x2_WAIT_(ta, off, ra, rb, kind) \
    do { \
    __syncwarp(); \
    asm volatile( \
        "{\n\t.reg .b32 tb;\n\tadd.u32 tb, %32, %33;\n\t" \
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t" \
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [tb];\n\t" \
        "tcgen05.wait::ld.sync.aligned;\n\t}" \
        : "=r"(ra[0]), "=r"(ra[1]), "=r"(ra[2]), "=r"(ra[3]), "=r"(ra[4]), "=r"(ra[5]), "=r"(ra[6]), \
          "=r"(ra[7]), "=r"(ra[8]), "=r"(ra[9]), "=r"(ra[10]), "=r"(ra[11]), "=r"(ra[12]), "=r"(ra[13]), \
          "=r"(ra[14]), "=r"(ra[15]), "=r"(rb[0]), "=r"(rb[1]), "=r"(rb[2]), "=r"(rb[3]), "=r"(rb[4]), \
          "=r"(rb[5]), "=r"(rb[6]), "=r"(rb[7]), "=r"(rb[8]), "=r"(rb[9]), "=r"(rb[10]), "=r"(rb[11]), \
          "=r"(rb[12]), "=r"(rb[13]), "=r"(rb[14]), "=r"(rb[15]) \
        : "r"(ta), kind(off) \
        : "memory"); \
    } while (0)
#define SSD_TMEM_ST16_WAIT(ta, ra) \
    do { \
    __syncwarp(); \
    asm volatile( \
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t" \
        "tcgen05.wait::st.sync.aligned;" \
        : \
        : "r"(ta), "r"(ra[0]), "r"(ra[1]), "r"(ra[2]), "r"(ra[3]), "r"(ra[4]), "r"(ra[5]), "r"(ra[6]), \
          "r"(ra[7]), "r"(ra[8]), "r"(ra[9]), "r"(ra[10]), "r"(ra[11]), "r"(ra[12]), "r"(ra[13]), "r"(ra[14]), \
          "r"(ra[15]) \
        : "memory"); \
    } while (0)
#define SSD_TMEM_ST16x2_WAIT(ta, ra, tb, rb) \
    do { \
    __syncwarp(); \
    asm volatile( \
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17};\n\t" \
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%1], {%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33};\n\t" \
        "tcgen05.wait::st.sync.aligned;" \
        : \
        : "r"(ta), "r"(tb), "r"(ra[0]), "r"(ra[1]), "r"(ra[2]), "r"(ra[3]), "r"(ra[4]), "r"(ra[5]), \
          "r"(ra[6]), "r"(ra[7]), "r"(ra[8]), "r"(ra[9]), "r"(ra[10]), "r"(ra[11]), "r"(ra[12]), \
          "r"(ra[13]), "r"(ra[14]), "r"(ra[15]), "r"(rb[0]), "r"(rb[1]), "r"(rb[2]), "r"(rb[3]), \
          "r"(rb[4]), "r"(rb[5]), "r"(rb[6]), "r"(rb[7]), "r"(rb[8]), "r"(rb[9]), "r"(rb[10]), "r"(rb[11]), \
          "r"(rb[12]), "r"(rb[13]), "r"(rb[14]), "r"(rb[15]) \
        : "memory"); \
    } while (0)

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// Byte offset of 16-byte chunk c (0..7) of row r inside a 128B-swizzled [rows][64 bf16] box.
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t c) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((c ^ (r & 7u)) << 4);
}

// Block-local inclusive prefix sum of a = dt*A over the 128 rows of one epilogue group.
// Every warp scans its quadrant's 32 rows; one warp per quadrant publishes the quadrant
// total and the group barrier orders it.  Returns cs for this row, the block total and
// the running totals at the end of each 32-row quadrant.
__device__ __forceinline__ float block_cumsum(float a, int q, int lane, bool publish, float* tot, int bar_id,
                                              float& cs_last, float* cend) {
    float v = a;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    if (publish && lane == 31) tot[q] = v;
    group_bar(bar_id);
    float pre = 0.f, run = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float tk = tot[k];
        if (k < q) pre += tk;
        run += tk;
        cend[k] = run;
    }
    cs_last = run;
    return v + pre;
}

// ------------------------------------------------------------------ kernel
// kRawDt: dt arrives raw (the DtMap pre-processing applies); it is then formed where a block
// uses it rather than where it is prefetched, so the prefetch still hides the load.
template <int kDecay, bool kRawDt = false>
__global__ void __launch_bounds__(kThreads, 1)
ssd_prefill_fused_kernel(const __grid_constant__ TcParams prm) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = prm.T, H = prm.H;
    // this CTA's work item: a whole unit, or one segment of a split unit
    int u, seg, nseg_u;
    if ((int)blockIdx.x < prm.n_full) {
        u = blockIdx.x, seg = 0, nseg_u = 1;
    } else {
        const int t = blockIdx.x - prm.n_full;
        u = prm.n_full + t / prm.nseg, seg = t % prm.nseg, nseg_u = prm.nseg;
    }
    const int hd = u % H, bi = u / H;
    const int g = hd / (H / prm.G);
    // this CTA's tokens: [tb, tb + span), in blocks of kBlk
    const int tb = seg * prm.tseg;
    const int nblk = ((nseg_u == 1 ? T : min(prm.tseg, T - tb)) + kBlk - 1) / kBlk;

    uint8_t* small = smem + kSmall;
    uint64_t* bars = reinterpret_cast<uint64_t*>(small);              // BAR_COUNT barriers
    // per-token decay terms of a block (two slots), published by the prep warp
    float* s_m = reinterpret_cast<float*>(small + 512);               // [2][128] log2(dt_j) - cs_j log2e
    float* s_v = s_m + 2 * kBlk;                                      // [2][128] exp(cs_e - cs_j) dt_j
    float* s_cs = s_v + 2 * kBlk;                                     // [2][128] cs_i
    float* s_w = s_cs + 2 * kBlk;                                     // [2][128] exp(cs_last - cs_j) dt_j
    float* s_cend = s_w + 2 * kBlk;                                   // [2][4] cs at the end of each 32-token group
    float* s_cslast = s_cend + 8;                                     // [2] the block's total log decay
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_cslast + 2);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_cslast + 4);

    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    if (threadIdx.x == 0) {
        const bool misaligned = (sbase & 1023u) != 0;  // swizzled layouts need a 1024-byte base
        if (misaligned) report_status(prm.status, SSD_ERR_INTERNAL | (1 << 8));
        for (int i = 0; i < BAR_COUNT; ++i) mbar_init(bar(i), bar_count(i));
        *s_abort = misaligned ? 1 : 0;
        s_wait_ns = prm.wait_ns;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const uint32_t tmem = tmem_alloc_cta(s_tmem, kTmemCols, warp == 1);  // warp 1 owns the TMEM
    if (tmem == kTmemSentinel) {
        *s_abort = 1;
        report_status(prm.status, SSD_ERR_INTERNAL | (3 << 8));
    }

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0 && !*s_abort && !prm.starve) {
            int issued = 0;
            for (int u = 0; u < nblk; ++u) {
                const int s2 = u & 1, s3 = u % 3;
                const int t0 = tb + u * kBlk;
                if (u >= 2 && !mbar_wait(bar(BAR_EMPTYCB + s2), ((u - 2) >> 1) & 1, s_abort, prm.status, 1)) break;
                const uint32_t fcb = bar(BAR_FULLCB + s2);
                const uint32_t slot = sbase + s2 * kCBSlot;
                mbar_expect_tx(fcb, 4 * kRegion);
                tma_load_4d(slot + kSlotC, &prm.tm_C, fcb, 0, g, t0, bi);
                tma_load_4d(slot + kSlotC + kRegion, &prm.tm_C, fcb, 64, g, t0, bi);
                tma_load_4d(slot + kSlotB, &prm.tm_B, fcb, 0, g, t0, bi);
                tma_load_4d(slot + kSlotB + kRegion, &prm.tm_B, fcb, 64, g, t0, bi);
                if (u >= 3 && !mbar_wait(bar(BAR_EMPTYX + s3), ((u - 3) / 3) & 1, s_abort, prm.status, 2)) {
                    issued = -(u + 1);  // C,B of block u issued, X not
                    break;
                }
                const uint32_t fx = bar(BAR_FULLX + s3);
                mbar_expect_tx(fx, kRegion);
                tma_load_4d(sbase + kXRing + s3 * kRegion, &prm.tm_x, fx, 0, hd, t0, bi);
                issued = u + 1;
            }
            // loads nobody may have waited for must land before the CTA exits
            const int ncb = issued < 0 ? -issued : issued;  // blocks whose C,B were issued
            const int nx = issued < 0 ? -issued - 1 : issued;
            for (int u = ncb - 2; u < ncb; ++u)
                if (u >= 0) mbar_drain(bar(BAR_FULLCB + (u & 1)), (u >> 1) & 1);
            for (int u = nx - 3; u < nx; ++u)
                if (u >= 0) mbar_drain(bar(BAR_FULLX + u % 3), (u / 3) & 1);
        }
    } else if (warp == 1) {
        // ================================================================ issuer 1: scores path
        // The whole warp runs this loop (operands stay warp-uniform); one elected lane issues
        // each tcgen05 instruction.
        constexpr uint32_t id_cb = idesc_bf16(128, 128, 0, 0);   // A C (K-major), B B (K-major)
        constexpr uint32_t id_y = idesc_bf16(128, 64, 0, 1);     // A P (TMEM), B X (MN-major)
        auto wt = [&](int b, uint32_t parity, int where) {
            return warp_wait(bar(b), parity, s_abort, prm.status, where);
        };
        auto issue_cb = [&](int k) {  // C B^T of block k (C, B in ring slot k & 1) into CB/P buffer k & 1
            const uint32_t slot = sbase + (k & 1) * kCBSlot;
            const uint64_t dC = sdesc(slot + kSlotC, 16, 1024), dB = sdesc(slot + kSlotB, 16, 1024);
            // a K step of 16 advances only the 16-byte address field of a K-major descriptor.
            // The K loops stay rolled: each tcgen05.mma site costs a few hundred bytes of code,
            // and instruction fetch, not issue rate, limits these warps
#pragma unroll 1
            for (int kk = 0; kk < kN / 16; ++kk) {
                const uint32_t off = (kk >> 2) * (kRegion >> 4) + (kk & 3) * 2;
                mma_ss_w(tmem + kColCBP + (k & 1) * 128, dC + off, dB + off, id_cb, kk > 0);
            }
            mma_commit_w(bar(BAR_CBFULL + (k & 1)));
            mma_commit_w(bar(BAR_EMPTYCB + (k & 1)));
        };
        auto issue_y = [&](int k) {  // Y = P_k X_k; P chunk c (K steps 2c, 2c+1) sits at column 32c
            const uint64_t dX = sdesc(sbase + kXRing + (k % 3) * kRegion, kRegion, 1024);
            const uint32_t pbuf = tmem + kColCBP + (k & 1) * 128;
#pragma unroll 1
            for (int kk = 0; kk < kBlk / 16; ++kk)
                mma_ts_w(tmem + kColY, pbuf + (kk >> 1) * 32 + (kk & 1) * 8, dX + kk * 128, id_y, kk > 0);
            mma_commit_w(bar(BAR_PXDONE + (k & 1)));
        };
        bool ok = __all_sync(0xffffffffu, !*s_abort);
        if (ok && nblk > 0) {
            ok = wt(BAR_FULLCB, 0, 3);
            if (ok) { tc_fence_after(); issue_cb(0); }
        }
        for (int k = 0; k < nblk && ok; ++k) {
            // C B^T of the next block first: the scores group's longest lead.  Its buffer was
            // last read by P X of block k - 1.
            if (k + 1 < nblk) {
                ok = wt(BAR_FULLCB + ((k + 1) & 1), ((k + 1) >> 1) & 1, 7) &&
                     (k < 1 || wt(BAR_PXDONE + ((k + 1) & 1), ((k - 1) >> 1) & 1, 4));
                if (!ok) break;
                tc_fence_after();
                issue_cb(k + 1);
            }
            // Y of block k: P written, X landed, and the scores group done reading Y of block k - 1
            ok = wt(BAR_PREADY + (k & 1), (k >> 1) & 1, 9) && wt(BAR_FULLX + k % 3, (k / 3) & 1, 8) &&
                 (k < 1 || wt(BAR_YFREE, (k - 1) & 1, 10));
            if (!ok) break;
            tc_fence_after();
            issue_y(k);
        }
        // every MMA and commit issued above completes before the TMEM is released
        mma_commit_w(bar(BAR_DONE1));
        mbar_drain(bar(BAR_DONE1), 0);
    } else if (warp == 2) {
        // ================================================================ issuer 2: state path
        constexpr uint32_t id_s = idesc_bf16(128, 64, 1, 1);     // A B^T (MN-major), B w o X (MN-major)
        constexpr uint32_t id_yst = idesc_bf16(128, 64, 0, 1);   // A C (K-major), B H^T (MN-major)
        auto wt = [&](int b, uint32_t parity, int where) {
            return warp_wait(bar(b), parity, s_abort, prm.status, where);
        };
        auto issue_s = [&](int k) {  // S_k^T = B^T (w o X)
            const uint32_t slot = sbase + (k & 1) * kCBSlot;
            const uint64_t dBt = sdesc(slot + kSlotB, kRegion, 1024), dXs = sdesc(sbase + kXs, kRegion, 1024);
#pragma unroll 1
            for (int kk = 0; kk < kBlk / 16; ++kk) mma_ss_w(tmem + kColS, dBt + kk * 128, dXs + kk * 128, id_s, kk > 0);
            mma_commit_w(bar(BAR_SDONE));
        };
        auto issue_yst = [&](int k) {  // C H_k^T into buffer k & 1; then C, B of block k are dead
            const uint32_t slot = sbase + (k & 1) * kCBSlot;
            const uint64_t dC = sdesc(slot + kSlotC, 16, 1024), dH = sdesc(sbase + kSH, kRegion, 1024);
#pragma unroll 1
            for (int kk = 0; kk < kN / 16; ++kk) {
                const uint32_t off = (kk >> 2) * (kRegion >> 4) + (kk & 3) * 2;
                mma_ss_w(tmem + kColYst + (k & 1) * 64, dC + off, dH + kk * 128, id_yst, kk > 0);  // MN step: 16 rows
            }
            mma_commit_w(bar(BAR_YSTDONE + (k & 1)));
            mma_commit_w(bar(BAR_EMPTYCB + (k & 1)));
        };
        bool ok = __all_sync(0xffffffffu, !*s_abort);
        for (int k = 0; k < nblk && ok; ++k) {
            // S of block k: C,B landed, w o X written, and S of block k - 1 read
            ok = wt(BAR_FULLCB + (k & 1), (k >> 1) & 1, 21) && wt(BAR_XSREADY, k & 1, 22) &&
                 (k < 1 || wt(BAR_SFREE, (k - 1) & 1, 23));
            if (!ok) break;
            tc_fence_after();
            issue_s(k);
            // C H^T of block k: H^T of the state entering block k written, and its buffer read
            // by the scores group for block k - 2
            ok = wt(BAR_HREADY, k & 1, 24) && (k < 2 || wt(BAR_YSTFREE + (k & 1), ((k - 2) >> 1) & 1, 25));
            if (!ok) break;
            tc_fence_after();
            issue_yst(k);
        }
        mma_commit_w(bar(BAR_DONE2));
        mbar_drain(bar(BAR_DONE2), 0);
    } else if (warp < kWarpState) {
        // ================================================================ scores group
        const int q = warp & 3, half = (warp - kWarpScores) >> 2;
        const int r = q * 32 + lane;  // token row i (and column index j for the per-token arrays)
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        const float Dh = prm.D[hd];
        const int p0 = half * 32;  // this warp's 32 of the 64 p columns of the output
        // y(k) = Y(k) + exp(cs_i) Yst(k) for row r, columns [p0, p0 + 32), into the swizzled
        // y tile in X slot k % 3: X(k) is dead once P X of block k is done and C H^T of block
        // k is done (the state group read X(k) for w o X before it published H^T(k), which
        // C H^T waited for).  The store warp writes the tile out with one TMA store.
        // exp(cs_i) is carried in a register: by now the state group may have republished
        // the arrays of block k's slot.
        auto store_y = [&](int k, float ei) {
            bool ok = warp_wait(bar(BAR_PXDONE + (k & 1)), (k >> 1) & 1, s_abort, prm.status, 12);
            if (ok) ok = warp_wait(bar(BAR_YSTDONE + (k & 1)), (k >> 1) & 1, s_abort, prm.status, 18);
            if (!ok) return false;
            tc_fence_after();
            uint32_t yp[16];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t ry[16], rs[16];
                const uint32_t ta = tmem + lane_addr + kColY + p0 + hh * 16;
                const uint32_t off = kColYst + (k & 1) * 64 - kColY;
                SSD_TMEM_LD16x2_WAIT_R(ta, off, ry, rs);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    yp[hh * 8 + j] = pack_bf16(fmaf(ei, __uint_as_float(rs[2 * j]), __uint_as_float(ry[2 * j])),
                                               fmaf(ei, __uint_as_float(rs[2 * j + 1]), __uint_as_float(ry[2 * j + 1])));
            }
            tc_fence_before();
            mbar_arrive(bar(BAR_YFREE));
            mbar_arrive(bar(BAR_YSTFREE + (k & 1)));
            uint8_t* dst = smem + kXRing + (k % 3) * kRegion;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                *reinterpret_cast<uint4*>(dst + swz(r, half * 4 + c4)) =
                    make_uint4(yp[4 * c4], yp[4 * c4 + 1], yp[4 * c4 + 2], yp[4 * c4 + 3]);
            fence_proxy_async();
            mbar_arrive(bar(BAR_YSTAGED + k % 3));
            return true;
        };
        bool live = __all_sync(0xffffffffu, !*s_abort);
        float ei_prev = 0.f;  // exp(cs_i) of the previous block
        for (int u = 0; u < nblk; ++u) {
            const int s = u & 1;
            const uint32_t buf = tmem + lane_addr + kColCBP + s * 128;
            float ei_cur = 0.f;
            // the state group publishes cs, the chunk ends and the per-column decay terms
            if (live) live = warp_wait(bar(BAR_PREP + s), (u >> 1) & 1, s_abort, prm.status, 17);
            if (live) live = warp_wait(bar(BAR_CBFULL + s), (u >> 1) & 1, s_abort, prm.status, 11);
            if (live) {
                // ---- P = bf16(CB o L) for this warp's chunks {half, half + 2} of row r,
                //      written over the first 16 of each chunk's 32 columns
                tc_fence_after();
                const float* vs = s_v + s * kBlk;
                const float* ms = s_m + s * kBlk;
                const float cs = s_cs[s * kBlk + r];
                const float csl = cs * kLog2e;
                ei_cur = dexp<kDecay>(__expf(cs));
                const float ce0 = s_cend[s * 4 + 0], ce1 = s_cend[s * 4 + 1], ce2 = s_cend[s * 4 + 2];
#pragma unroll 1
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = half + 2 * cc;
                    uint32_t pk[16];
                    if (c < q) {  // below the diagonal sub-block: factorised decay
                        uint32_t raw[32];
                        SSD_TMEM_LD32_WAIT(buf + c * 32, raw);
                        const float ce = (c == 0) ? ce0 : (c == 1) ? ce1 : ce2;
                        const float uu = dexp<kDecay>(__expf(cs - ce));
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float4 v4 = *reinterpret_cast<const float4*>(vs + c * 32 + 4 * k);
                            const float a0 = __uint_as_float(raw[4 * k + 0]) * uu;
                            const float a1 = __uint_as_float(raw[4 * k + 1]) * uu;
                            const float a2 = __uint_as_float(raw[4 * k + 2]) * uu;
                            const float a3 = __uint_as_float(raw[4 * k + 3]) * uu;
                            pk[2 * k] = pack_bf16(a0 * v4.x, a1 * v4.y);
                            pk[2 * k + 1] = pack_bf16(a2 * v4.z, a3 * v4.w);
                        }
                    } else if (c == q) {  // diagonal sub-block: per-element decay and causal mask
                        uint32_t raw[32];
                        SSD_TMEM_LD32_WAIT(buf + c * 32, raw);
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int j0 = 2 * k, j1 = 2 * k + 1;  // column within the sub-block
                            const float2 m2 = *reinterpret_cast<const float2*>(ms + c * 32 + j0);
                            float v0 = (j0 <= lane) ? __uint_as_float(raw[j0]) * dexp<kDecay>(ex2(csl + m2.x)) : 0.f;
                            float v1 = (j1 <= lane) ? __uint_as_float(raw[j1]) * dexp<kDecay>(ex2(csl + m2.y)) : 0.f;
                            if (j0 == lane) v0 += Dh;
                            if (j1 == lane) v1 += Dh;
                            pk[k] = pack_bf16(v0, v1);
                        }
                    } else {  // above the diagonal: zeros (the C B^T there is not read)
#pragma unroll
                        for (int k = 0; k < 16; ++k) pk[k] = 0u;
                    }
                    SSD_TMEM_ST16_WAIT(buf + c * 32, pk);
                }
                tc_fence_before();
                mbar_arrive(bar(BAR_PREADY + s));
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_ARRFREE + s));  // done with the block's decay terms
                // the previous block's output
                if (u >= 1) live = store_y(u - 1, ei_prev);
            }
            ei_prev = ei_cur;
        }
        // output of the last block
        if (live && nblk > 0) live = store_y(nblk - 1, ei_prev);
    } else if (warp < kWarpStore) {
        // ================================================================ state group
        const int q = warp & 3, half = (warp - kWarpState) >> 2;
        const int r = q * 32 + lane;  // token row (w o X) and state row n (S, H)
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        const int p0 = half * 32;  // this warp's 32 of the 64 p columns
        float Hs[32];              // fp32 running state H[p0 + k][r]
        if (seg == 0) {
            // state entering a whole unit or a first segment: h0
            const float* h0 = u < prm.n_full ? prm.h0 : prm.h0_split;
#pragma unroll
            for (int k = 0; k < 32; ++k) Hs[k] = h0 ? h0[(size_t)u * kP * kN + (size_t)(p0 + k) * kN + r] : 0.f;
        } else {
            // state entering segment seg: the end states of the segments before it, folded in
            // order, H <- exp(logdecay_q) H + H_q (already folded by the prefix pass when a
            // sequence has many segments).  This grid may start before the grid that wrote
            // them has ended.
            griddep_wait();
            const size_t o = (size_t)(u - prm.n_full) * (prm.nseg - 1);
            const float* st = prm.seg_state + o * kP * kN + r;
            const int first = prm.seg_prefix ? seg - 1 : 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) Hs[k] = st[(size_t)first * kP * kN + (size_t)(p0 + k) * kN];
#pragma unroll 1
            for (int q = first + 1; q < seg; ++q) {
                const float gq = __expf(prm.seg_logdecay[o + q]);
                const float* sq = st + (size_t)q * kP * kN;
                float v[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = sq[(size_t)(p0 + k) * kN];
#pragma unroll
                for (int k = 0; k < 32; ++k) Hs[k] = fmaf(gq, Hs[k], v[k]);
            }
        }
        auto write_sh = [&]() {  // bf16 H^T row r, chunks [4 half, 4 half + 4)
            uint8_t* dst = smem + kSH;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint4 v4;
                v4.x = pack_bf16(Hs[8 * c4 + 0], Hs[8 * c4 + 1]);
                v4.y = pack_bf16(Hs[8 * c4 + 2], Hs[8 * c4 + 3]);
                v4.z = pack_bf16(Hs[8 * c4 + 4], Hs[8 * c4 + 5]);
                v4.w = pack_bf16(Hs[8 * c4 + 6], Hs[8 * c4 + 7]);
                *reinterpret_cast<uint4*>(dst + swz(r, half * 4 + c4)) = v4;
            }
        };
        // H^T of the state entering block 0
        write_sh();
        fence_proxy_async();
        mbar_arrive(bar(BAR_HREADY));
        bool live = __all_sync(0xffffffffu, !*s_abort);
        float gam = 0.f;  // exp(total log decay) of the block whose S is folded in next
        // iteration j: fold S of block j into the state; w o X of block j+1; H^T of the state
        // entering block j+1
        for (int j = -1; j < nblk && live; ++j) {
            // ---- S of block j: read it, release the accumulator, H <- exp(cs_last(j)) H + S(j)
            if (j >= 0) {
                live = warp_wait(bar(BAR_SDONE), j & 1, s_abort, prm.status, 13);
                if (!live) break;
                tc_fence_after();
                uint32_t raw[32];
                SSD_TMEM_LD32_WAIT(tmem + lane_addr + kColS + p0, raw);
                tc_fence_before();
                mbar_arrive(bar(BAR_SFREE));
#pragma unroll
                for (int k = 0; k < 32; ++k) Hs[k] = fmaf(gam, Hs[k], __uint_as_float(raw[k]));
            }
            // ---- w o X of block j+1 (S of block j has read the previous w o X), with the
            //      weights w_j = exp(cs_last - cs_j) dt_j the prep warp published
            if (j + 1 < nblk) {
                const int s = (j + 1) & 1;
                live = warp_wait(bar(BAR_PREP + s), ((j + 1) >> 1) & 1, s_abort, prm.status, 16) &&
                       warp_wait(bar(BAR_FULLX + (j + 1) % 3), ((j + 1) / 3) & 1, s_abort, prm.status, 14);
                if (!live) break;
                const __nv_bfloat162 w2 = __float2bfloat162_rn(s_w[s * kBlk + r]);
                gam = dexp<kDecay>(__expf(s_cslast[s]));
                const uint8_t* src = smem + kXRing + ((j + 1) % 3) * kRegion;
                uint8_t* dst = smem + kXs;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int c = half * 4 + c4;
                    uint4 uv = *reinterpret_cast<const uint4*>(src + swz(r, c));
                    __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&uv);
#pragma unroll
                    for (int k = 0; k < 4; ++k) e[k] = __hmul2(e[k], w2);
                    *reinterpret_cast<uint4*>(dst + swz(r, c)) = uv;
                }
                fence_proxy_async();
                mbar_arrive(bar(BAR_XSREADY));
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_ARRFREE + s));  // done with the block's decay terms
            }
            // ---- bf16 H^T of the state entering block j+1, once C H^T of block j has read
            //      the previous one
            if (j >= 0 && j + 1 < nblk) {
                live = warp_wait(bar(BAR_YSTDONE + (j & 1)), (j >> 1) & 1, s_abort, prm.status, 15);
                if (!live) break;
                write_sh();
                fence_proxy_async();
                mbar_arrive(bar(BAR_HREADY));
            }
        }
        if (live && !*s_abort && prm.hf && seg == nseg_u - 1) {
            float* hf = prm.hf + ((size_t)bi * H + hd) * kP * kN;
#pragma unroll
            for (int j = 0; j < 32; ++j) hf[(size_t)(p0 + j) * kN + r] = Hs[j];
        }
    } else if (warp == kWarpPrep) {
        // ================================================================ prep warp
        // Per-token decay terms of every block, published two blocks ahead of their use: the
        // prefix sums cs of a = dt*A inside the block (lane l holds tokens l, 32+l, 64+l,
        // 96+l: four warp scans and the running chunk totals), and from them
        //   s_cs[i] = cs_i,  s_m[j] = log2(dt_j) - cs_j log2(e),  s_v[j] = exp(cs_e - cs_j) dt_j
        //   (e = the last token of j's 32-token group),  s_w[j] = exp(cs_last - cs_j) dt_j,
        //   s_cend = cs at the end of each group,  s_cslast = cs_last.
        const float Ah = prm.A[hd];
        const float dt_bias = (kRawDt && prm.dtm.bias) ? __ldg(prm.dtm.bias + hd) : 0.f;
        auto load4 = [&](int blk, float (&d)[4]) {  // dt as stored, 0 past the end
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int tok = tb + blk * kBlk + 32 * c + lane;
                d[c] = (blk < nblk && tok < T) ? __ldg(prm.dt + ((size_t)bi * T + tok) * H + hd) : 0.f;
            }
        };
        // dt is fetched three blocks ahead: it is a strided gather, and under full HBM load its
        // latency is microseconds
        float da[4], db[4], dc[4];
        load4(0, da);
        load4(1, db);
        load4(2, dc);
        bool live = __all_sync(0xffffffffu, !*s_abort);
        for (int blk = 0; blk < nblk && live; ++blk) {
            const int s = blk & 1;
            float dtv[4], cs[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int tok = tb + blk * kBlk + 32 * c + lane;
                dtv[c] = kRawDt ? (tok < T ? dt_softplus_clamp(da[c] + dt_bias, prm.dtm) : 0.f) : da[c];
                da[c] = db[c];
                db[c] = dc[c];
            }
            load4(blk + 3, dc);
            // inclusive prefix sums inside each 32-token group, then the running group totals
#pragma unroll
            for (int c = 0; c < 4; ++c) cs[c] = dtv[c] * Ah;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float o = __shfl_up_sync(0xffffffffu, cs[c], off);
                    if (lane >= off) cs[c] += o;
                }
            }
            float cend[4], run = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float tot = __shfl_sync(0xffffffffu, cs[c], 31);
                cs[c] = dlog<kDecay>(cs[c] + run);
                run += tot;
                cend[c] = dlog<kDecay>(run);
            }
            const float cs_last = cend[3];
            // the slot of block blk - 2 must have been read by the scores and state warps
            if (blk >= 2) live = warp_wait(bar(BAR_ARRFREE + s), ((blk - 2) >> 1) & 1, s_abort, prm.status, 19);
            if (!live) break;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int j = s * kBlk + 32 * c + lane;
                s_cs[j] = cs[c];
                s_m[j] = __log2f(dtv[c]) - cs[c] * kLog2e;  // -inf where dt = 0
                s_v[j] = dexp<kDecay>(__expf(cend[c] - cs[c])) * dtv[c];
                s_w[j] = dexp<kDecay>(__expf(cs_last - cs[c])) * dtv[c];
            }
            if (lane < 4) s_cend[s * 4 + lane] = lane == 0 ? cend[0] : lane == 1 ? cend[1] : lane == 2 ? cend[2] : cend[3];
            if (lane == 0) s_cslast[s] = cs_last;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BAR_PREP + s));
        }
    } else if (warp == kWarpStore) {
        // ================================================================ y-store warp
        // One lane writes each block's y tile with a TMA store once the scores group has
        // staged it, waits until the store has read the tile out of shared memory, and
        // returns the X slot to the producer.
        if (lane == 0 && !*s_abort) {
            for (int k = 0; k < nblk; ++k) {
                const int s3 = k % 3;
                if (!mbar_wait(bar(BAR_YSTAGED + s3), (k / 3) & 1, s_abort, prm.status, 20)) break;
                tma_store_4d(sbase + kXRing + s3 * kRegion, &prm.tm_y, 0, hd, tb + k * kBlk, bi);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(bar(BAR_EMPTYX + s3));
            }
            // the stores must be complete before the CTA's shared memory goes away
            bulk_wait0();
        }
    }

    // ================================================================ teardown
    // Both issuers have seen their final commits land and the producer its last loads; only
    // then is the TMEM released.  The grid ends after the one before it in the stream.
    griddep_wait();
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == 1 && tmem != kTmemSentinel) {
        tc_fence_after();
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ------------------------------------------------------------------ segment state pass
// For a sequence split into segments, the state a segment leaves behind when it starts
// from zero ("Chunked recurrence" run over the segment alone) and the segment's total log
// decay sum(dt*A); the first segment's end state starts from h0.  Folding the earlier
// segments' end states in order gives every later segment its entering state (the fused
// kernel does that itself, or the prefix pass below when there are many segments).
// One CTA per segment of kHP heads of one sequence that share a B/C group: with kHP = 2 the
// group's B tile is loaded once for both heads and one MMA (N = 128) serves both, which cuts
// the bytes a block moves from 48 KB per head to 32 KB.
//
// The local state is the decayed sum over the segment's tokens,
//   H_loc = sum_j exp(cs_end - cs_j) dt_j x_j B_j^T,
// which the kernel evaluates as ONE tcgen05 accumulation over the whole segment: each
// block's tokens are weighted straight to the segment end, so no state is carried,
// rescaled or read back block by block.  Blocks are walked from the last to the first so
// that the log decay from a block's end to the segment's end (`later`, the sum of the
// totals of the blocks already walked) is known when the block arrives.  The weights
// underflow only where exp(cs_end - cs_j) itself underflows fp32, as in the block-by-block
// recurrence.
//
//   warp 0       TMA producer: B (two 64-column boxes) and the X of each head of a block
//                into ring slot u % kSlots (u counts blocks in walking order)
//   warp 1       TMEM owner and MMA issuer: S^T += B^T (w o X), N = 64 kHP (the heads' X
//                tiles side by side); each block's completion frees its slot
//   warps 2-9    state group: block prefix sums, w o X in place over X in the slot (one
//                head per half of the group when kHP = 2); at the end S^T out of TMEM to
//                the segment-state buffer
constexpr int kSThreads = 64 + kGroupThreads;
constexpr uint32_t kSX = 2 * kRegion;                // X tiles follow the two B regions
template <int kHP>
struct SPass {
    static constexpr uint32_t kSlot = (2 + kHP) * kRegion;  // B (n 0..63, 64..127), then X per head
    static constexpr int kSlots = kHP == 1 ? 2 : 3;          // 96 KB or 192 KB of loads in flight
    static constexpr uint32_t kSmall = kSlots * kSlot;
    static constexpr uint32_t kSmem = kSmall + 1024;
    static constexpr uint32_t kTmemCols = 64 * kHP;          // fp32 S^T accumulators (128 n x 64 p each)
    static constexpr int kMinBlocks = kHP == 1 ? 2 : 1;      // CTAs per SM
};
static_assert(SPass<1>::kSmem * 2 <= 232448 && SPass<2>::kSmem <= 232448, "state pass shared memory");
enum { SB_FULL = 0, SB_EMPTY = 3, SB_XS = 6, SB_ACC = 9, SB_DONE = 10, SB_COUNT };

template <int kDecay, int kHP>
__global__ void __launch_bounds__(kSThreads, SPass<kHP>::kMinBlocks)
ssd_segment_state_kernel(const __grid_constant__ TcParams prm) {
    using SP = SPass<kHP>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = prm.T, H = prm.H;
    // this CTA: segment seg (not the last) of split units su0 .. su0 + kHP - 1 (heads
    // hd0 .. hd0 + kHP - 1 of one sequence, in one group)
    const int su0 = (blockIdx.x / (prm.nseg - 1)) * kHP, seg = blockIdx.x % (prm.nseg - 1);
    const int u0 = prm.n_full + su0;
    const int hd0 = u0 % H, bi = u0 / H;
    const int g = hd0 / (H / prm.G);
    const int tb = seg * prm.tseg;
    const int nblk = (min(prm.tseg, T - tb) + kBlk - 1) / kBlk;
    // token offset of the u-th block walked (last block first)
    auto block_t0 = [&](int u) { return tb + (nblk - 1 - u) * kBlk; };

    uint8_t* small = smem + SP::kSmall;
    uint64_t* bars = reinterpret_cast<uint64_t*>(small);
    float* s_tot = reinterpret_cast<float*>(small + 128);          // [2][kHP][4] quadrant sums
    volatile int* s_abort = reinterpret_cast<volatile int*>(small + 192);
    volatile int* s_ystop = s_abort + 1;                           // [2]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(small + 208);
    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    if (threadIdx.x == 0) {
        const bool misaligned = (sbase & 1023u) != 0;
        if (misaligned) report_status(prm.status, SSD_ERR_INTERNAL | (2 << 8));
        for (int i = 0; i < SB_COUNT; ++i) mbar_init(bar(i), (i >= SB_XS && i < SB_XS + 3) ? kGroupThreads : 1);
        *s_abort = misaligned ? 1 : 0;
        s_wait_ns = prm.wait_ns;
        s_ystop[0] = s_ystop[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const uint32_t tmem = tmem_alloc_cta(s_tmem, SP::kTmemCols, warp == 1);  // warp 1 owns the TMEM
    if (tmem == kTmemSentinel) {
        *s_abort = 1;
        report_status(prm.status, SSD_ERR_INTERNAL | (4 << 8));
    }
    // the fused pass may be scheduled now: only its segments after the first read what this
    // grid writes, and they wait for it to end
    griddep_launch();
    constexpr int kS = SP::kSlots;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0 && !*s_abort && !prm.starve) {
            int issued = 0;
            for (int u = 0; u < nblk; ++u) {
                // slot u % kS is free once the MMAs of block u - kS have read it
                if (u >= kS && !mbar_wait(bar(SB_EMPTY + u % kS), ((u - kS) / kS) & 1, s_abort, prm.status, 40)) break;
                const uint32_t f = bar(SB_FULL + u % kS);
                const uint32_t slot = sbase + (u % kS) * SP::kSlot;
                const int t0 = block_t0(u);
                mbar_expect_tx(f, (2 + kHP) * kRegion);
                tma_load_4d(slot, &prm.tm_B, f, 0, g, t0, bi);
                tma_load_4d(slot + kRegion, &prm.tm_B, f, 64, g, t0, bi);
#pragma unroll
                for (int h = 0; h < kHP; ++h) tma_load_4d(slot + kSX + h * kRegion, &prm.tm_x, f, 0, hd0 + h, t0, bi);
                issued = u + 1;
            }
            for (int u = issued - kS; u < issued; ++u)
                if (u >= 0) mbar_drain(bar(SB_FULL + u % kS), (u / kS) & 1);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        // A B^T (MN-major), B the heads' w o X tiles (MN-major, 64-column atoms a region apart)
        constexpr uint32_t id_s = idesc_bf16(128, 64 * kHP, 1, 1);
        auto wt = [&](int b, uint32_t parity, int where) {
            return warp_wait(bar(b), parity, s_abort, prm.status, where);
        };
        bool ok = __all_sync(0xffffffffu, !*s_abort);
        for (int u = 0; u < nblk && ok; ++u) {
            ok = wt(SB_FULL + u % kS, (u / kS) & 1, 41) && wt(SB_XS + u % kS, (u / kS) & 1, 42);
            if (!ok) break;
            tc_fence_after();
            const uint32_t slot = sbase + (u % kS) * SP::kSlot;
            const uint64_t dBt = sdesc(slot, kRegion, 1024), dXs = sdesc(slot + kSX, kRegion, 1024);
#pragma unroll 1
            for (int kk = 0; kk < kBlk / 16; ++kk)
                mma_ss_w(tmem, dBt + kk * 128, dXs + kk * 128, id_s, (u > 0 || kk > 0) ? 1u : 0u);
            mma_commit_w(bar(SB_EMPTY + u % kS));
        }
        // the accumulator is complete (or, on the abort path, abandoned) once every MMA issued
        // above has landed; the drain keeps the TMEM alive until then
        mma_commit_w(bar(SB_ACC));
        mma_commit_w(bar(SB_DONE));
        mbar_drain(bar(SB_DONE), 0);
    } else {
        // ================================================================ state group
        const int q = warp & 3, half = (warp - 2) >> 2;
        const int r = q * 32 + lane;  // token row of a block (w o X) and state row n (S)
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        // kHP = 1: both halves on the one head, 32 of its 64 p columns each;
        // kHP = 2: half h takes head hd0 + h, all 64 columns
        const int h = kHP == 2 ? half : 0;
        const int hd = hd0 + h;
        constexpr int kChunks = 8 / (3 - kHP);  // 16-byte chunks of an X row per thread: 4 or 8
        const int c0 = kHP == 2 ? 0 : half * 4;
        const float Ah = prm.A[hd];
        // dt as stored (raw when the DtMap pre-processing applies), fetched two blocks ahead and
        // formed where the block uses it, so the prefetch is never waited on early
        auto load_dt = [&](int u) {
            const int tok = block_t0(u) + r;
            return (u < nblk && tok < T) ? __ldg(prm.dt + ((size_t)bi * T + tok) * H + hd) : 0.f;
        };
        bool live = __all_sync(0xffffffffu, !*s_abort);
        bool stopped = false;
        float dt_a = load_dt(0), dt_b = load_dt(1);
        const float dt_bias = (prm.dtm.raw && prm.dtm.bias) ? __ldg(prm.dtm.bias + hd) : 0.f;  // loaded once
        float later = 0.f;  // log decay from the end of the current block to the end of the segment
        for (int u = 0; u < nblk; ++u) {
            const int s = u & 1;  // stop-flag and quadrant-sum buffer
            const float dtv =
                block_t0(u) + r < T ? (prm.dtm.raw ? dt_softplus_clamp(dt_a + dt_bias, prm.dtm) : dt_a) : 0.f;
            dt_a = dt_b;
            dt_b = load_dt(u + 2);
            if (!live || *s_abort) s_ystop[s] = 1;
            float cend[4], cs_last;
            float cs = block_cumsum(dtv * Ah, q, lane, kHP == 2 || half == 0, s_tot + (s * kHP + h) * 4, 4, cs_last,
                                    cend);
            cs = dlog<kDecay>(cs);
            cs_last = dlog<kDecay>(cs_last);
            if (s_ystop[s]) {
                stopped = true;
                break;
            }
            if (live) {
                live = warp_wait(bar(SB_FULL + u % kS), (u / kS) & 1, s_abort, prm.status, 44);
                if (live) {
                    // w_j x_j in place with w_j = exp(cs_end - cs_j) dt_j, one packed bf16x2
                    // multiply per element pair
                    const __nv_bfloat162 w2 = __float2bfloat162_rn(dexp<kDecay>(__expf(later + cs_last - cs)) * dtv);
                    uint8_t* xs = smem + (u % kS) * SP::kSlot + kSX + h * kRegion;
#pragma unroll
                    for (int c4 = 0; c4 < kChunks; ++c4) {
                        uint4 uv = *reinterpret_cast<const uint4*>(xs + swz(r, c0 + c4));
                        __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&uv);
#pragma unroll
                        for (int j = 0; j < 4; ++j) e[j] = __hmul2(e[j], w2);
                        *reinterpret_cast<uint4*>(xs + swz(r, c0 + c4)) = uv;
                    }
                    fence_proxy_async();
                    mbar_arrive(bar(SB_XS + u % kS));
                }
            }
            later += cs_last;
        }
        // H_loc^T row n = r of head hd, this thread's p columns, out of the accumulator
        if (!stopped && live) live = warp_wait(bar(SB_ACC), 0, s_abort, prm.status, 45);
        if (!stopped && live) {
            tc_fence_after();
            constexpr int kCols = 32 * kHP;  // 32 (half of one head) or 64 (a whole head)
            const int pbase = kHP == 2 ? 0 : half * 32;
            uint32_t raw[kCols];
            if constexpr (kHP == 2) {
                uint32_t* raw_hi = raw + 32;
                SSD_TMEM_LD32x2_WAIT(tmem + lane_addr + h * 64, 32, raw, raw_hi);
            } else {
                SSD_TMEM_LD32_WAIT(tmem + lane_addr + h * 64 + pbase, raw);
            }
            tc_fence_before();
            if (!*s_abort) {
                const size_t o = (size_t)(su0 + h) * (prm.nseg - 1) + seg;
                float* dst = prm.seg_state + o * kP * kN;
                if (seg == 0 && prm.h0) {
                    // the first segment's end state starts from h0: exp(logdecay) h0 + H_loc
                    const float gam = __expf(later);
                    const float* h0 = prm.h0 + (size_t)(u0 + h) * kP * kN;
#pragma unroll
                    for (int j = 0; j < kCols; ++j) {
                        const size_t e = (size_t)(pbase + j) * kN + r;
                        dst[e] = fmaf(gam, h0[e], __uint_as_float(raw[j]));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < kCols; ++j) dst[(size_t)(pbase + j) * kN + r] = __uint_as_float(raw[j]);
                }
                if (r == 0 && (kHP == 2 || half == 0)) prm.seg_logdecay[o] = later;
            }
        }
    }

    griddep_wait();  // the grid ends after the one before it in the stream
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (warp == 1 && tmem != kTmemSentinel) {
        tc_fence_after();
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(SP::kTmemCols));
    }
}

int sm_count();

// Clears the status word ahead of a prefill and lets the prefill's first grid start at once
// (that grid's writes to the word wait for this one).
__global__ void ssd_status_reset_kernel(int* status) {
    if (threadIdx.x == 0) *status = 0;
    griddep_launch();
}

// Launches `k` with programmatic stream serialization: it may start while the grid ahead of
// it in the stream still runs, and waits (griddep_wait) where it needs that grid's results.
template <typename Param>
cudaError_t launch_pdl(void (*k)(Param), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                       const Param& prm) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, prm);
}

int reset_status(int* status, cudaStream_t s) {
    if (const int st = smem_limit_once((const void*)ssd_status_reset_kernel, 0)) return st;
    {
        LaunchScope ls("ssd_status_reset", s);
        ssd_status_reset_kernel<<<1, 32, 0, s>>>(status);
    }
    SSD_CUDA_TRY(cudaGetLastError());
    return SSD_OK;
}

// Launches the state pass over the split units [n_full, n_full + n_split): two heads per CTA
// where both heads of every pair share a B/C group, one otherwise.
template <int kHP>
int launch_state_pass_hp(const TcParams& prm, int decay, unsigned grid, cudaStream_t s) {
    auto k = decay == 1 ? ssd_segment_state_kernel<1, kHP>
             : decay == 2 ? ssd_segment_state_kernel<2, kHP>
                          : ssd_segment_state_kernel<0, kHP>;
    if (const int st = smem_limit_once((const void*)k, (int)SPass<kHP>::kSmem)) return st;
    {
        LaunchScope ls("ssd_segment_state", s);
        SSD_CUDA_TRY(launch_pdl(k, grid, kSThreads, SPass<kHP>::kSmem, s, prm));
    }
    return SSD_OK;
}
int launch_state_pass(const TcParams& prm, int n_split, int decay, cudaStream_t s) {
    // a pair (u, u + 1) starts at an even head, so both heads sit in one group when the
    // group size is even; the split units must then pair up exactly.  Pairs run one CTA per
    // SM, so they are used only when their grid fills the GPU (else two single-head CTAs per
    // SM spread the work wider).
    const bool pair = (prm.H / prm.G) % 2 == 0 && prm.n_full % 2 == 0 && n_split % 2 == 0 &&
                      (double)(n_split / 2) * (prm.nseg - 1) >= sm_count();
    const unsigned grid = (unsigned)((size_t)(n_split / (pair ? 2 : 1)) * (prm.nseg - 1));
    return pair ? launch_state_pass_hp<2>(prm, decay, grid, s) : launch_state_pass_hp<1>(prm, decay, grid, s);
}

// Folding kernel geometry: each (sequence, head) state is spread over kScanSplit CTAs; a
// thread carries kScanPer entries through the stretches, loading kScanBatch stretches'
// worth before the dependent updates.
constexpr int kScanSplit = 8, kScanThreads = 128, kScanPer = kP * kN / (kScanSplit * kScanThreads), kScanBatch = 4;

// Prefix pass over a split unit's segment end states, in place: H_q <- exp(logdecay_q)
// H_{q-1} + H_q for q = 1 .. nseg - 2, so that H_q becomes the state entering segment q + 1
// (H_0 already starts from h0).  Used when a sequence has more segments than the fused
// kernel folds itself; the same operations in the same order as that fold.
__global__ void __launch_bounds__(kScanThreads) ssd_segment_prefix_kernel(float* seg_state, const float* seg_logdecay,
                                                                           int nseg) {
    griddep_launch();  // the fused pass may be scheduled; its later segments wait for this grid
    griddep_wait();    // the state pass's end states
    const size_t o = (size_t)blockIdx.x * (nseg - 1);
    float* st = seg_state + o * kP * kN + blockIdx.z * (kP * kN / kScanSplit) + threadIdx.x;
    float run[kScanPer];
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) run[k] = st[kScanThreads * k];
    for (int q0 = 1; q0 + 1 < nseg; q0 += kScanBatch) {
        float v[kScanBatch][kScanPer], gam[kScanBatch];
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
            const bool in = q0 + j + 1 < nseg;
            gam[j] = in ? __expf(seg_logdecay[o + q0 + j]) : 0.f;
#pragma unroll
            for (int k = 0; k < kScanPer; ++k) v[j][k] = in ? st[(size_t)(q0 + j) * kP * kN + kScanThreads * k] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
            if (q0 + j + 1 >= nseg) break;
#pragma unroll
            for (int k = 0; k < kScanPer; ++k) {
                run[k] = fmaf(gam[j], run[k], v[j][k]);
                st[(size_t)(q0 + j) * kP * kN + kScanThreads * k] = run[k];
            }
        }
    }
}

// Folds consecutive stretches of one sequence into one state, per (sequence, head) u:
// run = h0 (or 0); for q in [0, n): run = exp(logdecay_q) run + h_q; out = run, and
// out_logdecay = sum of logdecay_q (when given).  Stretch q of unit u = bi * H + hd sits at
// st + q * st_q + u * st_u (P x N fp32), its log decay at ld + q * ld_q + u * ld_u (strides
// in elements).  Serves the context-parallel prefill (the stretches: the ranks before this
// one, rank-major) and the local state of a stretch computed in pieces (unit-major).
__global__ void __launch_bounds__(kScanThreads) ssd_state_fold_kernel(const float* h0, const float* st, size_t st_q,
                                                                       size_t st_u, const float* ld, size_t ld_q,
                                                                       size_t ld_u, int n, int H, float* out,
                                                                       float* out_logdecay) {
    const int hd = blockIdx.x, bi = blockIdx.y;
    const size_t u = (size_t)bi * H + hd;
    const int e0 = blockIdx.z * (kP * kN / kScanSplit) + threadIdx.x;
    float run[kScanPer];
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) run[k] = h0 ? h0[u * kP * kN + e0 + kScanThreads * k] : 0.f;
    float ldsum = 0.f;
    for (int q0 = 0; q0 < n; q0 += kScanBatch) {
        float v[kScanBatch][kScanPer], gam[kScanBatch];
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
            const bool in = q0 + j < n;
            const float l = in ? ld[(q0 + j) * ld_q + u * ld_u] : 0.f;
            ldsum += l;
            gam[j] = __expf(l);
            const float* w = st + (q0 + j) * st_q + u * st_u;
#pragma unroll
            for (int k = 0; k < kScanPer; ++k) v[j][k] = in ? w[e0 + kScanThreads * k] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
            if (q0 + j >= n) break;
#pragma unroll
            for (int k = 0; k < kScanPer; ++k) run[k] = fmaf(gam[j], run[k], v[j][k]);
        }
    }
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) out[u * kP * kN + e0 + kScanThreads * k] = run[k];
    if (out_logdecay && blockIdx.z == 0 && threadIdx.x == 0) out_logdecay[u] = ldsum;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D bf16 tensor map over [d3][d2][d1][d0] (d0 contiguous) with a {64, 1, 128, 1} box.
int make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3) {
    auto enc = get_encoder();
    if (!enc) return set_error(SSD_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[4] = {d0, d1, d2, d3};
    cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kBlk, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(SSD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SSD_OK;
}

}  // namespace

bool prefill_tc_supported(int P, int N, int io) { return io == SSD_BF16 && P == kP && N == kN; }

namespace {
constexpr size_t kSegOffset = 512;  // status word and launch scratch come first
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// SMs of the device current at the first call (148 when no device answers); initialised
// once, thread-safely
int sm_count() {
    static const int n = [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            v <= 0)
            v = 148;
        return v;
    }();
    return n;
}

// How the fused pass splits its work.  One CTA walks a unit's (or a segment's) blocks
// one after another, so the fused pass costs about (blocks per CTA) x (waves of CTAs)
// block-times when the waves are full and about (all blocks / SMs) when CTAs of a ragged
// last wave finish early; the model takes the mean of the two; a CTA's start (TMEM
// allocation, first loads) costs about two more block-times.  Splitting units into
// segments adds CTAs where b * H alone leaves SMs idle -- all units when b * H is below
// the SM count, or only the units of a ragged last wave -- at the price of the state pass
// (two CTAs per SM, measured at about 0.7 of a fused block-time per block), the fold of the
// segment states (about 0.4 block-times per segment) and a fixed cost for the extra launch.
// The cheapest candidate wins, but only where it beats the unsplit pass by 5 %.  Splitting only the units of a ragged
// last wave is priced from its own measurements instead: the state pass then runs beside
// the first wave of whole units (the fused grid may start as soon as the state pass runs),
// and costs about 1.5 block-times per extra segment plus one; that split is taken when it
// pays by 3 %.
struct SplitPlan {
    int n_full, nseg, tseg;  // see TcParams
};
constexpr double kStatePassPerBlock = 0.7;  // single-head state pass; the paired one measures ~0.5
constexpr double kCtaStartBlocks = 2.0;
constexpr double kScanPerSegment = 0.4;
constexpr double kSplitFixedBlocks = 5.0;
constexpr double kTailSplitPerSegment = 1.5, kTailSplitFixed = 1.0;
constexpr int kFoldMax = 5;  // the fused kernel folds up to this many segment states itself
std::atomic<int> g_force_nseg{0};     // 0: cost model
std::atomic<int> g_force_nfull{-1};   // -1: every unit split when nseg > 1
std::atomic<int> g_decay_mode{0};

// mean of the wave and flow estimates for `ctas` CTAs of `len` block-times
double pass_cost(double ctas, double len, double sms) {
    if (ctas <= 0) return 0.0;
    return 0.5 * (std::ceil(ctas / sms) * len + std::max(ctas * len / sms, len));
}

SplitPlan plan_split(int b, int T, int H) {
    const int nb = (T + kBlk - 1) / kBlk;
    const int units = b * H;
    SplitPlan none{units, 1, nb * kBlk};
    auto with_segments = [&](int n_full, int n) {
        const int bps = (nb + n - 1) / n;
        return SplitPlan{n_full, (nb + bps - 1) / bps, bps * kBlk};
    };
    if (const int f = g_force_nseg.load()) {
        const int n = std::min(f, nb);
        if (n <= 1) return none;
        const int nf = g_force_nfull.load();
        return with_segments(nf < 0 ? 0 : std::min(nf, units), n);
    }
    const double sms = sm_count();
    const double whole = pass_cost(units, nb + kCtaStartBlocks, sms);
    SplitPlan best = none;
    double best_cost = whole;
    // candidates: split every unit, or only the units past the last whole wave
    const int full_waves = (units / (int)sms) * (int)sms;
    for (const int n_full : {0, full_waves}) {
        if (n_full >= units || (n_full == full_waves && n_full == 0 && full_waves != 0)) continue;
        const double r = units - n_full;
        for (int bps = nb - 1; bps >= 1; --bps) {
            const int n = (nb + bps - 1) / bps;
            // of the lengths that give n segments only the shortest (the most even split) counts
            if (bps > 1 && (nb + bps - 2) / (bps - 1) == n) continue;
            const double len = bps + kCtaStartBlocks;
            double cost = (n_full ? std::ceil(n_full / sms) * (nb + kCtaStartBlocks) : 0.0) + pass_cost(r * n, len, sms);
            if (n_full)
                cost += kTailSplitPerSegment * (n - 1) + kTailSplitFixed;
            else
                cost += kStatePassPerBlock * std::ceil(r * (n - 1) / (2.0 * sms)) * len + kScanPerSegment * n +
                        kSplitFixedBlocks;
            if (cost < (n_full ? 0.97 : 0.95) * whole && cost < best_cost) {
                best_cost = cost;
                best = SplitPlan{n_full, n, bps * kBlk};
            }
        }
    }
    return best;
}
}  // namespace

int prefill_tc_segments(int b, int T, int H) { return plan_split(b, T, H).nseg; }
int prefill_tc_whole_units(int b, int T, int H) {
    const SplitPlan sp = plan_split(b, T, H);
    return sp.nseg == 1 ? b * H : sp.n_full;
}

// Workspace: the status word, then (split sequences only) the segments' end states, their
// log decays, and room for a copy of h0 for when h0 and h_final are one buffer.  The fused
// kernel reads that copy at the same unit offsets as h0, and the copy holds the split units
// [n_full, b*H) only, so its room spans all b*H units.
struct SplitLayout {
    size_t state, logdecay, h0copy, bytes;
};
SplitLayout split_layout(int b, int H, const SplitPlan& sp) {
    const size_t n_split = (size_t)(b * H - sp.n_full), units = n_split * (sp.nseg - 1);
    SplitLayout l;
    l.state = kSegOffset;
    l.logdecay = l.state + align256(units * kP * kN * sizeof(float));
    l.h0copy = l.logdecay + align256(units * sizeof(float));
    l.bytes = l.h0copy + align256((size_t)b * H * kP * kN * sizeof(float));
    return l;
}

size_t prefill_tc_workspace_bytes(int b, int T, int H) {
    const SplitPlan sp = plan_split(b, T, H);
    if (sp.nseg == 1) return kSegOffset;
    return split_layout(b, H, sp).bytes;
}

namespace {
std::atomic<unsigned long long> g_starve_ns{0};
}
void prefill_tc_starve_next(unsigned long long wait_ns) { g_starve_ns.store(wait_ns); }
void prefill_tc_force_segments(int nseg) {
    g_force_nfull.store(-1);
    g_force_nseg.store(nseg);
}
void prefill_tc_force_split(int n_full, int nseg) {
    g_force_nfull.store(n_full);
    g_force_nseg.store(nseg);
}
void prefill_tc_decay_mode(int mode) { g_decay_mode.store(mode); }

int launch_prefill_tc(int b, int T, int H, int G, const void* x, const float* dt, const DtMap& dtm, const float* A,
                      const void* Bm,
                      const void* Cm, const float* D, const float* h0, void* y, float* hf, void* ws,
                      cudaStream_t s) {
    TcParams prm;
    memset(&prm, 0, sizeof(prm));
    int st;
    if ((st = make_map(&prm.tm_x, x, kP, H, T, b)) != SSD_OK) return st;
    if ((st = make_map(&prm.tm_B, Bm, kN, G, T, b)) != SSD_OK) return st;
    if ((st = make_map(&prm.tm_C, Cm, kN, G, T, b)) != SSD_OK) return st;
    if ((st = make_map(&prm.tm_y, y, kP, H, T, b)) != SSD_OK) return st;
    prm.dt = dt;
    prm.dtm = dtm;
    const int decay = g_decay_mode.load();
    auto fused = dtm.raw ? (decay == 1   ? ssd_prefill_fused_kernel<1, true>
                            : decay == 2 ? ssd_prefill_fused_kernel<2, true>
                                         : ssd_prefill_fused_kernel<0, true>)
                         : (decay == 1   ? ssd_prefill_fused_kernel<1, false>
                            : decay == 2 ? ssd_prefill_fused_kernel<2, false>
                                         : ssd_prefill_fused_kernel<0, false>);
    prm.A = A;
    prm.D = D;
    prm.h0 = h0;
    prm.hf = hf;
    prm.y = static_cast<__nv_bfloat16*>(y);
    prm.status = reinterpret_cast<int*>(ws);
    prm.T = T;
    prm.H = H;
    prm.G = G;
    const SplitPlan sp = plan_split(b, T, H);
    prm.n_full = sp.n_full;
    prm.nseg = sp.nseg;
    prm.tseg = sp.tseg;
    const int n_split = b * H - sp.n_full;
    prm.h0_split = h0;
    if (prm.nseg > 1) {
        const SplitLayout l = split_layout(b, H, sp);
        char* w = static_cast<char*>(ws);
        prm.seg_state = reinterpret_cast<float*>(w + l.state);
        prm.seg_logdecay = reinterpret_cast<float*>(w + l.logdecay);
        if (h0 && h0 == hf) {
            // the first segment of a split unit reads h0 from a copy: the unit's last segment
            // overwrites h0 with h_final, and nothing orders the two CTAs
            float* cp = reinterpret_cast<float*>(w + l.h0copy);
            const size_t off = (size_t)sp.n_full * kP * kN;
            SSD_CUDA_TRY(cudaMemcpyAsync(cp + off, h0 + off, (size_t)n_split * kP * kN * sizeof(float),
                                         cudaMemcpyDeviceToDevice, s));
            prm.h0_split = cp;
        }
    }
    const unsigned long long starve_ns = g_starve_ns.exchange(0);
    prm.starve = starve_ns != 0;
    prm.wait_ns = starve_ns ? starve_ns : kWaitLimitNs;
    // Grids in a row, each allowed to start before the one ahead ends: the status reset; for
    // split sequences the end states of all segments but the last, and when there are many
    // segments their prefix pass; the fused pass, whose later segments fold in the end states
    // (or read the prefix) once the grid before has ended
    prm.seg_prefix = prm.nseg - 1 > kFoldMax;
    if ((st = reset_status(prm.status, s)) != SSD_OK) return st;
    if (prm.nseg > 1 && (st = launch_state_pass(prm, n_split, decay, s)) != SSD_OK) return st;
    if (prm.seg_prefix) {
        if ((st = smem_limit_once((const void*)ssd_segment_prefix_kernel, 0)) != SSD_OK) return st;
        LaunchScope ls("ssd_segment_prefix", s);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)n_split, 1, kScanSplit);
        cfg.blockDim = dim3(kScanThreads);
        cfg.stream = s;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        SSD_CUDA_TRY(cudaLaunchKernelEx(&cfg, ssd_segment_prefix_kernel, prm.seg_state,
                                        (const float*)prm.seg_logdecay, prm.nseg));
    }
    if ((st = smem_limit_once((const void*)fused, (int)kSmemBytes)) != SSD_OK) return st;
    {
        LaunchScope ls("ssd_prefill_fused", s);
        SSD_CUDA_TRY(launch_pdl(fused, (unsigned)(prm.n_full + (size_t)n_split * prm.nseg), kThreads, kSmemBytes, s, prm));
    }
    return SSD_OK;
}

// Local end state of a stretch of tokens started from zero, and its total log decay (the
// context-parallel prefill's first step).  The stretch is cut into pieces so that the
// state pass fills the SMs; the pieces' states are then folded in order.
namespace {
int local_pieces(int b, int T, int H) {
    const int nb = (T + kBlk - 1) / kBlk;
    const int want = (int)std::ceil(4.0 * sm_count() / std::max(1.0, (double)b * H));  // two waves of 2 CTAs/SM
    return std::max(1, std::min(nb, want));
}
}  // namespace

size_t prefill_tc_local_state_workspace_bytes(int b, int T, int H) {
    const int n = local_pieces(b, T, H);
    const size_t units = (size_t)b * H * n;
    return kSegOffset + align256(units * kP * kN * sizeof(float)) + align256(units * sizeof(float));
}

int launch_prefill_tc_local_state(int b, int T, int H, int G, const void* x, const float* dt, const float* A,
                                  const void* Bm, float* h_local, float* log_decay, void* ws, cudaStream_t s) {
    TcParams prm;
    memset(&prm, 0, sizeof(prm));
    int st;
    if ((st = make_map(&prm.tm_x, x, kP, H, T, b)) != SSD_OK) return st;
    if ((st = make_map(&prm.tm_B, Bm, kN, G, T, b)) != SSD_OK) return st;
    prm.dt = dt;
    prm.dtm = DtMap{nullptr, 0.f, 0.f, 0};
    prm.A = A;
    prm.status = reinterpret_cast<int*>(ws);
    prm.T = T;
    prm.H = H;
    prm.G = G;
    const int n = local_pieces(b, T, H);
    const int nb = (T + kBlk - 1) / kBlk;
    prm.tseg = ((nb + n - 1) / n) * kBlk;
    const int pieces = (T + prm.tseg - 1) / prm.tseg;
    prm.n_full = 0;
    prm.nseg = pieces + 1;  // the state pass writes pieces 0 .. nseg-2, i.e. every piece
    const size_t units = (size_t)b * H * pieces;
    prm.seg_state = reinterpret_cast<float*>(static_cast<char*>(ws) + kSegOffset);
    prm.seg_logdecay = reinterpret_cast<float*>(static_cast<char*>(ws) + kSegOffset +
                                                align256(units * kP * kN * sizeof(float)));
    prm.wait_ns = kWaitLimitNs;
    if ((st = reset_status(prm.status, s)) != SSD_OK) return st;
    if ((st = launch_state_pass(prm, b * H, 0, s)) != SSD_OK) return st;
    // piece q of unit u: state at (u * pieces + q) * P * N, log decay at u * pieces + q
    {
        LaunchScope ls("ssd_state_fold", s);
        ssd_state_fold_kernel<<<dim3(H, b, kScanSplit), kScanThreads, 0, s>>>(
            nullptr, prm.seg_state, (size_t)kP * kN, (size_t)pieces * kP * kN, prm.seg_logdecay, 1, (size_t)pieces,
            pieces, H, h_local, log_decay);
    }
    SSD_CUDA_TRY(cudaGetLastError());
    return SSD_OK;
}

// Entering state of context shard `rank` from the gathered local states and log decays of
// all shards, rank-major ([world][b][H][P][N], [world][b][H]).
int launch_context_scan(int rank, int b, int H, const float* h0, const float* h_all, const float* ld_all,
                        float* h_in, cudaStream_t s) {
    LaunchScope ls("ssd_state_fold", s);
    ssd_state_fold_kernel<<<dim3(H, b, kScanSplit), kScanThreads, 0, s>>>(
        h0, h_all, (size_t)b * H * kP * kN, (size_t)kP * kN, ld_all, (size_t)b * H, 1, rank, H, h_in, nullptr);
    SSD_CUDA_TRY(cudaGetLastError());
    return SSD_OK;
}

// Reads and clears the device status word the fused kernel writes on a failed wait.
int prefill_tc_status(void* ws, cudaStream_t s) {
    int v = 0;
    SSD_CUDA_TRY(cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s));
    SSD_CUDA_TRY(cudaStreamSynchronize(s));
    if (v == 0) return SSD_OK;
    SSD_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(int), s));
    const int code = v & 0xff, where = v >> 8;
    if (code == SSD_ERR_INTERNAL) {
        const char* what = where == 1   ? "fused kernel: dynamic shared memory not 1024-byte aligned"
                           : where == 2 ? "segment state pass: dynamic shared memory not 1024-byte aligned"
                           : where == 3 ? "fused kernel: tensor-memory address never arrived"
                           : where == 4 ? "segment state pass: tensor-memory address never arrived"
                                        : "unknown check";
        return set_error(code, "device consistency check %d failed (%s)", where, what);
    }
    return set_error(code, "device status %d at wait site %d", code, where);
}

}  // namespace ssd
