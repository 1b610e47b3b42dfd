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
//   warp 0       TMA producer: C, B (two 64-column 128B-swizzled boxes each) and X per
//                block into two stages
//   warp 1       TMEM owner and MMA issuer (one lane), per block t:
//                  CB(t+1) = C B^T        (M=128 i, N=128 j, K=128 n)   SS   -> TMEM
//                  S(t)^T  = B^T (w o X)  (M=128 n, N=64 p,  K=128 j)   SS   -> TMEM
//                  Y(t)    = P X          (M=128 i, N=64 p,  K=128 j)   TS (P in TMEM)
//                  Yst(t)  = C H^T        (M=128 i, N=64 p,  K=128 n)   SS
//   warps 2-9    "scores" group (2 warps per TMEM lane quadrant): prefix sum of dt*A,
//                w o X into shared memory, and the decayed causal scores P = bf16(CB o L)
//                written back into TMEM as the A operand of the next MMA
//   warps 10-17  "state" group (2 warps per quadrant): H <- exp(cs_last) H + S (fp32,
//                registers), bf16 H^T for the next C H^T, y = Y + exp(cs_i) Yst, TMA store
// The scores group runs one block ahead of the state group, so the tensor core, the TMA
// engine and both epilogues overlap.
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
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace ssd {
namespace {

constexpr int kBlk = 128;    // tokens per block = MMA M
constexpr int kP = 64;       // head dim
constexpr int kN = 128;      // state size
constexpr int kGroupThreads = 256;  // threads per epilogue group
constexpr int kThreads = 64 + 2 * kGroupThreads;
constexpr float kLog2e = 1.4426950408889634f;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t kRegion = kBlk * 128;             // one [128 rows][64 bf16] swizzled box: 16 KB
constexpr uint32_t kStageC = 0;                      // 2 regions (n 0..63, 64..127)
constexpr uint32_t kStageB = 2 * kRegion;            // 2 regions
constexpr uint32_t kStageX = 4 * kRegion;            // 1 region
constexpr uint32_t kStageBytes = 5 * kRegion;        // 80 KB
constexpr uint32_t kXs = 2 * kStageBytes;            // two w o X buffers
constexpr uint32_t kSH = kXs + 2 * kRegion;          // bf16 H^T [n][p]
constexpr uint32_t kYst = kSH + kRegion;             // y staging tile for the TMA store
constexpr uint32_t kSmall = kYst + kRegion;          // barriers and per-token scalars
constexpr uint32_t kSmallBytes = 2560;
constexpr uint32_t kSmemBytes = kSmall + kSmallBytes;
constexpr uint32_t kTxBytes = 5 * kRegion;           // bytes landing per stage
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns (512 x 128 lanes x 32 bit)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColCB = 0;      // two 128-column fp32 C B^T buffers; S(t) reuses buffer t%2
constexpr uint32_t kColP = 256;     // bf16 scores, 2 per column (64 columns)
constexpr uint32_t kColY = 320;     // two 64-column Y buffers
constexpr uint32_t kColYst = 448;   // 64 columns

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

// barrier indices in the small area
enum {
    BAR_FULL0 = 0, BAR_FULL1, BAR_EMPTY0, BAR_EMPTY1, BAR_CB0, BAR_CB1, BAR_ACCS0, BAR_ACCS1,
    BAR_SCORES, BAR_PFREE, BAR_SFREE, BAR_ACCY, BAR_H, BAR_DONE, BAR_COUNT
};

struct TcParams {
    CUtensorMap tm_x;
    CUtensorMap tm_B;
    CUtensorMap tm_C;
    CUtensorMap tm_y;
    const float* dt;
    const float* A;
    const float* D;
    const float* h0;
    float* hf;
    int* status;
    int T, H, G, nblk;
};

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
// Bounded wait for the phase with `parity` to complete.  Returns false (and makes every
// other role give up) if the CTA is aborting or the limit expires.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, int where) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicCAS(status, 0, SSD_ERR_TIMEOUT | (where << 8));
            return false;
        }
    }
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
    while (!mbar_try(bar, parity) && globaltimer() - t0 < kWaitLimitNs) {
    }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* tm, uint32_t src, int c0, int c1, int c2, int c3) {
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
__device__ __forceinline__ void group_bar(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kGroupThreads) : "memory");
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

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
__device__ __forceinline__ void mma_ss(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
        ::"r"(tmem_d), "r"(tmem_a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

#define SSD_TMEM_LD32(taddr, r)                                                                          \
    asm volatile(                                                                                        \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15," \
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                      \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),           \
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),        \
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),     \
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),     \
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])                                              \
        : "r"(taddr))
#define SSD_TMEM_LD16(taddr, r)                                                                          \
    asm volatile(                                                                                        \
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}," \
        " [%16];"                                                                                        \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),           \
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),        \
          "=r"(r[14]), "=r"(r[15])                                                                        \
        : "r"(taddr))
#define SSD_TMEM_ST16(taddr, r)                                                                          \
    asm volatile(                                                                                        \
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"  \
        "%15,%16};"                                                                                      \
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),      \
          "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),   \
          "r"(r[15])                                                                                      \
        : "memory")
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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
__global__ void __launch_bounds__(kThreads, 1)
ssd_prefill_fused_kernel(const __grid_constant__ TcParams prm) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hd = blockIdx.x, bi = blockIdx.y;
    const int T = prm.T, H = prm.H, nblk = prm.nblk;
    const int g = hd / (H / prm.G);

    uint8_t* small = smem + kSmall;
    uint64_t* bars = reinterpret_cast<uint64_t*>(small);              // BAR_COUNT barriers
    float* s_m = reinterpret_cast<float*>(small + 128);               // [2][128] log2(dt_j) - cs_j log2e
    float* s_v = s_m + 2 * kBlk;                                      // [2][128] exp(cs_e - cs_j) dt_j
    float* s_stot = s_v + 2 * kBlk;                                   // [2][4] scores-group quadrant sums
    float* s_ytot = s_stot + 8;                                       // [2][4] state-group quadrant sums
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_ytot + 8);
    volatile int* s_sstop = s_abort + 1;                              // [2]
    volatile int* s_ystop = s_abort + 3;                              // [2]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_ytot + 16);

    const uint32_t sbase = smem_u32(smem);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    if (threadIdx.x == 0) {
        const bool misaligned = (sbase & 1023u) != 0;  // swizzled layouts need a 1024-byte base
        if (misaligned) atomicCAS(prm.status, 0, SSD_ERR_INTERNAL | (1 << 8));
        mbar_init(bar(BAR_FULL0), 1);
        mbar_init(bar(BAR_FULL1), 1);
        mbar_init(bar(BAR_EMPTY0), 1);
        mbar_init(bar(BAR_EMPTY1), 1);
        mbar_init(bar(BAR_CB0), 1);
        mbar_init(bar(BAR_CB1), 1);
        mbar_init(bar(BAR_ACCS0), 1);
        mbar_init(bar(BAR_ACCS1), 1);
        mbar_init(bar(BAR_SCORES), kGroupThreads);
        mbar_init(bar(BAR_PFREE), 1);
        mbar_init(bar(BAR_SFREE), kGroupThreads);
        mbar_init(bar(BAR_ACCY), 1);
        mbar_init(bar(BAR_H), kGroupThreads);
        mbar_init(bar(BAR_DONE), 1);
        *s_abort = misaligned ? 1 : 0;
        s_sstop[0] = s_sstop[1] = 0;
        s_ystop[0] = s_ystop[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // TMEM allocation (whole warp)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0 && !*s_abort) {
            int issued = 0;
            for (int t = 0; t < nblk; ++t) {
                const int s = t & 1;
                if (t >= 2 && !mbar_wait(bar(BAR_EMPTY0 + s), ((t - 2) >> 1) & 1, s_abort, prm.status, 1)) break;
                const uint32_t full = bar(BAR_FULL0 + s);
                const uint32_t st = sbase + s * kStageBytes;
                mbar_expect_tx(full, kTxBytes);
                const int t0 = t * kBlk;
                tma_load_4d(st + kStageC, &prm.tm_C, full, 0, g, t0, bi);
                tma_load_4d(st + kStageC + kRegion, &prm.tm_C, full, 64, g, t0, bi);
                tma_load_4d(st + kStageB, &prm.tm_B, full, 0, g, t0, bi);
                tma_load_4d(st + kStageB + kRegion, &prm.tm_B, full, 64, g, t0, bi);
                tma_load_4d(st + kStageX, &prm.tm_x, full, 0, hd, t0, bi);
                issued = t + 1;
            }
            // the last (up to) two stages may hold loads nobody waited for: let them land
            for (int u = issued - 2; u < issued; ++u)
                if (u >= 0) mbar_drain(bar(BAR_FULL0 + (u & 1)), (u >> 1) & 1);
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0 && !*s_abort) {
            constexpr uint32_t id_cb = idesc_bf16(128, 128, 0, 0);   // A C (K-major), B B (K-major)
            constexpr uint32_t id_s = idesc_bf16(128, 64, 1, 1);     // A B^T (MN-major), B w o X (MN-major)
            constexpr uint32_t id_y = idesc_bf16(128, 64, 0, 1);     // A P (TMEM), B X (MN-major)
            constexpr uint32_t id_yst = idesc_bf16(128, 64, 0, 1);   // A C (K-major), B H^T (MN-major)
            auto issue_cb = [&](int u) {
                const uint32_t st = sbase + (u & 1) * kStageBytes;
                const uint32_t d = tmem + kColCB + (u & 1) * 128;
#pragma unroll
                for (int k = 0; k < kN / 16; ++k) {
                    const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
                    mma_ss(d, sdesc(st + kStageC + off, 16, 1024), sdesc(st + kStageB + off, 16, 1024), id_cb, k > 0);
                }
                mma_commit(bar(BAR_CB0 + (u & 1)));
            };
            bool ok = mbar_wait(bar(BAR_FULL0), 0, s_abort, prm.status, 2);
            if (ok) {
                tc_fence_after();
                issue_cb(0);
            }
            for (int t = 0; t < nblk && ok; ++t) {
                const int s = t & 1;
                const uint32_t st = sbase + s * kStageBytes;
                // (a) C B^T of the next block, into the buffer whose S was consumed
                if (t + 1 < nblk) {
                    if (!(ok = mbar_wait(bar(BAR_FULL0 + (s ^ 1)), ((t + 1) >> 1) & 1, s_abort, prm.status, 3))) break;
                    if (t >= 1 && !(ok = mbar_wait(bar(BAR_SFREE), (t - 1) & 1, s_abort, prm.status, 4))) break;
                    tc_fence_after();
                    issue_cb(t + 1);
                }
                // (b) S(t)^T = B^T (w o X) into buffer s; Y(t) = P X
                if (!(ok = mbar_wait(bar(BAR_SCORES), t & 1, s_abort, prm.status, 5))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kBlk / 16; ++k)
                    mma_ss(tmem + kColCB + s * 128, sdesc(st + kStageB + k * 2048, kRegion, 1024),
                           sdesc(sbase + kXs + s * kRegion + k * 2048, kRegion, 1024), id_s, k > 0);
                mma_commit(bar(BAR_ACCS0 + s));
#pragma unroll
                for (int k = 0; k < kBlk / 16; ++k)
                    mma_ts(tmem + kColY + s * 64, tmem + kColP + k * 8, sdesc(st + kStageX + k * 2048, kRegion, 1024),
                           id_y, k > 0);
                mma_commit(bar(BAR_PFREE));
                // (c) Yst(t) = C H_t^T
                if (!(ok = mbar_wait(bar(BAR_H), t & 1, s_abort, prm.status, 6))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kN / 16; ++k) {
                    const uint32_t offa = (k >> 2) * kRegion + (k & 3) * 32;
                    mma_ss(tmem + kColYst, sdesc(st + kStageC + offa, 16, 1024),
                           sdesc(sbase + kSH + k * 2048, kRegion, 1024), id_yst, k > 0);
                }
                mma_commit(bar(BAR_ACCY));
                mma_commit(bar(BAR_EMPTY0 + s));
            }
            // every MMA and commit issued above completes before the TMEM is released
            mma_commit(bar(BAR_DONE));
            mbar_drain(bar(BAR_DONE), 0);
        }
    } else if (warp < 10) {
        // ================================================================ scores group
        const int q = warp & 3, half = (warp - 2) >> 2;
        const int r = q * 32 + lane;  // token row i (and column index j for the per-token arrays)
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        const float Ah = prm.A[hd], Dh = prm.D[hd];
        bool live = __all_sync(0xffffffffu, !*s_abort);
        for (int t = 0; t < nblk; ++t) {
            const int s = t & 1;
            const int t0 = t * kBlk;
            // ---- prefix sums; per-token arrays for block t (slot s)
            const float dtv = (t0 + r < T) ? prm.dt[((size_t)bi * T + t0 + r) * H + hd] : 0.f;
            if (!live || *s_abort) s_sstop[s] = 1;
            float cend[4], cs_last;
            const float cs = block_cumsum(dtv * Ah, q, lane, half == 0, s_stot + s * 4, 2, cs_last, cend);
            if (s_sstop[s]) break;  // identical for the whole group (read after its barrier)
            if (half == 0) {
                s_m[s * kBlk + r] = __log2f(dtv) - cs * kLog2e;                 // -inf where dt = 0
                s_v[s * kBlk + r] = __expf(cend[q] - cs) * dtv;                  // cend[q]: end of j's quadrant
            }
            group_bar(2);
            const float w = __expf(cs_last - cs) * dtv;

            // ---- w o X into Xs[s] (row r = token j; this warp's 4 of the 8 chunks)
            if (live) live = warp_wait(bar(BAR_FULL0 + s), (t >> 1) & 1, s_abort, prm.status, 7);
            if (live && t >= 2) live = warp_wait(bar(BAR_ACCS0 + s), ((t - 2) >> 1) & 1, s_abort, prm.status, 8);
            if (live) {
                const uint8_t* src = smem + s * kStageBytes + kStageX;
                uint8_t* dst = smem + kXs + s * kRegion;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int c = half * 4 + c4;
                    uint4 u = *reinterpret_cast<const uint4*>(src + swz(r, c));
                    uint32_t* e = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&e[k]));
                        e[k] = pack_bf16(f.x * w, f.y * w);
                    }
                    *reinterpret_cast<uint4*>(dst + swz(r, c)) = u;
                }
            }
            // ---- P = bf16(CB o L) for this warp's chunks {half, half + 2} of row r
            if (live) live = warp_wait(bar(BAR_CB0 + s), (t >> 1) & 1, s_abort, prm.status, 9);
            if (live) {
                tc_fence_after();
                const float* vs = s_v + s * kBlk;
                const float* ms = s_m + s * kBlk;
                const float csl = cs * kLog2e;
                bool pfree_seen = (t == 0);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = half + 2 * cc;
                    uint32_t pk[16];
                    if (c < q) {  // below the diagonal sub-block: factorised decay
                        uint32_t raw[32];
                        SSD_TMEM_LD32(tmem + lane_addr + kColCB + s * 128 + c * 32, raw);
                        const float u = __expf(cs - cend[c]);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float4 v4 = *reinterpret_cast<const float4*>(vs + c * 32 + 4 * k);
                            const float a0 = __uint_as_float(raw[4 * k + 0]) * u;
                            const float a1 = __uint_as_float(raw[4 * k + 1]) * u;
                            const float a2 = __uint_as_float(raw[4 * k + 2]) * u;
                            const float a3 = __uint_as_float(raw[4 * k + 3]) * u;
                            pk[2 * k] = pack_bf16(a0 * v4.x, a1 * v4.y);
                            pk[2 * k + 1] = pack_bf16(a2 * v4.z, a3 * v4.w);
                        }
                    } else if (c == q) {  // diagonal sub-block: per-element decay and causal mask
                        uint32_t raw[32];
                        SSD_TMEM_LD32(tmem + lane_addr + kColCB + s * 128 + c * 32, raw);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int j0 = 2 * k, j1 = 2 * k + 1;  // column within the sub-block
                            const float2 m2 = *reinterpret_cast<const float2*>(ms + c * 32 + j0);
                            float v0 = (j0 <= lane) ? __uint_as_float(raw[j0]) * ex2(csl + m2.x) : 0.f;
                            float v1 = (j1 <= lane) ? __uint_as_float(raw[j1]) * ex2(csl + m2.y) : 0.f;
                            if (j0 == lane) v0 += Dh;
                            if (j1 == lane) v1 += Dh;
                            pk[k] = pack_bf16(v0, v1);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k) pk[k] = 0u;
                    }
                    if (!pfree_seen) {  // the previous block's P X must be done reading P
                        live = warp_wait(bar(BAR_PFREE), (t - 1) & 1, s_abort, prm.status, 10);
                        pfree_seen = true;
                        if (!live) break;
                        tc_fence_after();
                    }
                    SSD_TMEM_ST16(tmem + lane_addr + kColP + c * 16, pk);
                }
                if (live) tmem_wait_st();
            }
            fence_proxy_async();
            tc_fence_before();
            if (live) mbar_arrive(bar(BAR_SCORES));
        }
    } else {
        // ================================================================ state group
        const int q = warp & 3, half = (warp - 10) >> 2;
        const int r = q * 32 + lane;  // state row n (state update) and token row i (output)
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        const float Ah = prm.A[hd];
        const size_t hbase = ((size_t)bi * H + hd) * kP * kN;
        const int p0 = half * 32;  // this warp's 32 of the 64 p columns
        float Hs[32];              // fp32 running state H[p0 + k][r]
#pragma unroll
        for (int k = 0; k < 32; ++k) Hs[k] = prm.h0 ? prm.h0[hbase + (size_t)(p0 + k) * kN + r] : 0.f;
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
        write_sh();
        fence_proxy_async();
        mbar_arrive(bar(BAR_H));
        bool live = __all_sync(0xffffffffu, !*s_abort);
        bool stopped = false;
        const bool leader = (warp == 10 && lane == 0);
        for (int t = 0; t < nblk; ++t) {
            const int s = t & 1;
            const int t0 = t * kBlk;
            const float dtv = (t0 + r < T) ? prm.dt[((size_t)bi * T + t0 + r) * H + hd] : 0.f;
            if (!live || *s_abort) s_ystop[s] = 1;
            float cend[4], cs_last;
            const float cs = block_cumsum(dtv * Ah, q, lane, half == 0, s_ytot + s * 4, 3, cs_last, cend);
            if (s_ystop[s]) { stopped = true; break; }
            const float gam = __expf(cs_last);
            const float ei = __expf(cs);

            // ---- H <- exp(cs_last) H + S(t)   (S(t)^T lives in C B^T buffer s)
            if (live) live = warp_wait(bar(BAR_ACCS0 + s), (t >> 1) & 1, s_abort, prm.status, 11);
            if (live) {
                tc_fence_after();
                uint32_t raw[32];
                SSD_TMEM_LD32(tmem + lane_addr + kColCB + s * 128 + p0, raw);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) Hs[k] = fmaf(gam, Hs[k], __uint_as_float(raw[k]));
                tc_fence_before();
                mbar_arrive(bar(BAR_SFREE));
            }
            // ---- y(t) = Y(t) + exp(cs_i) Yst(t); then hand H_{t+1} to the next C H^T
            uint32_t yp[16];
            if (live) live = warp_wait(bar(BAR_ACCY), t & 1, s_abort, prm.status, 12);
            if (live) {
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t ry[16], rs[16];
                    SSD_TMEM_LD16(tmem + lane_addr + kColY + s * 64 + p0 + hh * 16, ry);
                    SSD_TMEM_LD16(tmem + lane_addr + kColYst + p0 + hh * 16, rs);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        yp[hh * 8 + k] = pack_bf16(fmaf(ei, __uint_as_float(rs[2 * k]), __uint_as_float(ry[2 * k])),
                                                   fmaf(ei, __uint_as_float(rs[2 * k + 1]), __uint_as_float(ry[2 * k + 1])));
                }
                write_sh();  // C H_t^T (read by Yst(t)) has completed
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(bar(BAR_H));
            }
            // ---- stage y(t) and store it with TMA
            if (leader) bulk_wait_read0();  // the previous tile has left the staging buffer
            group_bar(3);
            if (live) {
                uint8_t* dst = smem + kYst;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4)
                    *reinterpret_cast<uint4*>(dst + swz(r, half * 4 + c4)) =
                        make_uint4(yp[4 * c4], yp[4 * c4 + 1], yp[4 * c4 + 2], yp[4 * c4 + 3]);
            }
            fence_proxy_async();
            if (!live || *s_abort) s_ystop[s ^ 1] = 1;
            group_bar(3);
            if (leader && !s_ystop[s ^ 1]) {
                tma_store_4d(&prm.tm_y, sbase + kYst, 0, hd, t0, bi);
                bulk_commit();
            }
        }
        if (leader) bulk_wait0();
        if (!stopped && live && !*s_abort && prm.hf) {
#pragma unroll
            for (int k = 0; k < 32; ++k) prm.hf[hbase + (size_t)(p0 + k) * kN + r] = Hs[k];
        }
    }

    // ================================================================ teardown
    // The MMA lane has seen its final commit land, the producer its last loads, and the
    // state group its y stores; only then is the TMEM released.
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
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

size_t prefill_tc_workspace_bytes() { return 256; }

int launch_prefill_tc(int b, int T, int H, int G, const void* x, const float* dt, const float* A, const void* Bm,
                      const void* Cm, const float* D, const float* h0, void* y, float* hf, void* ws,
                      cudaStream_t s) {
    TcParams prm;
    memset(&prm, 0, sizeof(prm));
    int st;
    if ((st = make_map(&prm.tm_x, x, kP, H, T, b)) != SSD_OK) return st;
    if ((st = make_map(&prm.tm_y, y, kP, H, T, b)) != SSD_OK) return st;
    if ((st = make_map(&prm.tm_B, Bm, kN, G, T, b)) != SSD_OK) return st;
    if ((st = make_map(&prm.tm_C, Cm, kN, G, T, b)) != SSD_OK) return st;
    prm.dt = dt;
    prm.A = A;
    prm.D = D;
    prm.h0 = h0;
    prm.hf = hf;
    prm.status = reinterpret_cast<int*>(ws);
    prm.T = T;
    prm.H = H;
    prm.G = G;
    prm.nblk = (T + kBlk - 1) / kBlk;
    SSD_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(int), s));
    SSD_CUDA_TRY(cudaFuncSetAttribute(ssd_prefill_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kSmemBytes));
    {
        LaunchScope ls("ssd_prefill_fused", s);
        ssd_prefill_fused_kernel<<<dim3(H, b), kThreads, kSmemBytes, s>>>(prm);
    }
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
    return set_error(code, "device status %d at wait site %d", code, where);
}

}  // namespace ssd
