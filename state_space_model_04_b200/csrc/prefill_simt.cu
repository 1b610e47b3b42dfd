// prefill_simt.cu -- chunked SSD prefill on CUDA cores (fp32 FMA), four kernels that
// follow the method's steps one to one.
//
// Method: "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching"
// (arXiv 2603.09555): the dual form over chunks of L tokens (Eq. 3) with the decay
// matrix exp(cs_i - cs_j) (j <= i) from a segment-wise prefix sum of A*dt ("Diagonal
// state matrix" property), chunk summary states, a sequential recurrence over them
// ("Chunked recurrence" property), the state-to-output term and the D skip.
//
//   K1 (inside K2)    cs = inclusive prefix sum of a = dt*A inside each chunk
//   K2 chunk_state    S_c[p][n] = sum_j exp(cs_last - cs_j) dt_j x_j[p] B_j[n], as partial
//                     sums over slices of the chunk's tokens (one CTA per slice)
//   K3 state_scan     S_c = the slices' partials summed in order; H_0 = h0,
//                     H_{c+1} = exp(cs_last(c)) H_c + S_c  (in place: S -> H_in)
//   K4 chunk_output   y_i = sum_{j<=i} (C_i.B_j) exp(cs_i-cs_j) dt_j x_j
//                           + exp(cs_i) C_i.H_c + D x_i
// When (chunks x heads x sequences) alone would leave most SMs idle, the chunk state is
// split over slices of 32 tokens and the output over 16-row tiles whose products are split
// into four quarters of their contraction; partial states and quarters are added in a fixed
// order, so results are bitwise reproducible from run to run.  The two output kernels sum in
// different orders, so a batch size that moves a call from one to the other changes y by
// rounding only.
//
// This path serves fp32 inputs: every product and sum is an fp32 FMA (no TF32), and the
// prefix sums are kept in fp64 (CsT = double) so that exp(cs_i - cs_j) keeps full fp32
// accuracy even when |cs| reaches several hundred inside a chunk.  A ragged last chunk
// is handled as if padded with dt = 0 tokens, which leave the state unchanged.
#include <algorithm>
#include <cmath>
#include <type_traits>

#include "common.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kP = 64;

// exp of a (non-positive) log-space decay difference, rounded to fp32.  fp64 prefix sums
// are exponentiated in fp64 so the fp32 path keeps full accuracy.
__device__ __forceinline__ float exp_cs(double v) { return (float)exp(v); }
__device__ __forceinline__ float exp_cs(float v) { return expf(v); }

// Runs `count` (a multiple of the block size) element copies through registers, eight per
// thread at a time: the group's global loads are all in flight before its stores.
template <int kCount, typename Load, typename Store>
__device__ __forceinline__ void copy_grouped(Load load, Store store) {
    constexpr int kPer = kCount / kThreads, kGrp = kPer < 8 ? kPer : 8;
    static_assert(kCount % kThreads == 0 && kPer % kGrp == 0, "tile size");
#pragma unroll 1
    for (int k0 = 0; k0 < kPer; k0 += kGrp) {
        float r[kGrp];
#pragma unroll
        for (int k = 0; k < kGrp; ++k) r[k] = load(threadIdx.x + (k0 + k) * kThreads);
#pragma unroll
        for (int k = 0; k < kGrp; ++k) store(threadIdx.x + (k0 + k) * kThreads, r[k]);
    }
}

// Asynchronous 4-byte global -> shared copy (zero fill when !valid; src is then not read).
__device__ __forceinline__ void cp_async4(float* dst, const float* src, bool valid) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory"); }

// Copies a kRows x W tile (row r at src + r * stride, W contiguous elements; rows r >= valid
// are zeros) into float shared memory, element (r, c) at dst[r * ld + c] or, transposed, at
// dst[c * ld + r]: asynchronously for fp32 inputs, through registers (converting) for bf16.
// A thread keeps one column c and walks rows kThreads / W apart, so each element costs one
// pointer step.
template <int W, int kRows, bool kTransposed, typename IoT>
__device__ __forceinline__ void tile_load(float* dst, int ld, const IoT* src, size_t stride, int valid) {
    static_assert(kThreads % W == 0 && kRows * W % kThreads == 0, "tile size");
    constexpr int kStep = kThreads / W;  // rows between a thread's elements
    const int c = threadIdx.x % W, r0 = threadIdx.x / W;
    const IoT* s = src + r0 * stride + c;
    const size_t s_step = kStep * stride;
    float* d = kTransposed ? dst + c * ld + r0 : dst + r0 * ld + c;
    const int d_step = kTransposed ? kStep : kStep * ld;
#pragma unroll
    for (int k = 0; k < kRows / kStep; ++k) {
        const bool v = r0 + k * kStep < valid;
        if constexpr (std::is_same<IoT, float>::value) {
            cp_async4(d, v ? s : src, v);
        } else {
            *d = v ? load_io(s, 0) : 0.f;
        }
        s += s_step;
        d += d_step;
    }
}

// ---------------------------------------------------------------- K1 + K2
// One CTA per (slice of chunk c, head, sequence).  Every CTA forms its chunk's prefix sums
// with one block scan (L <= 256 = the CTA's threads); the CTAs of slice 0 store them for K3
// and K4.  A CTA then accumulates the tokens of its slices -- [32 sl, 32 sl + 32), then
// every ks-th slice after it -- into its own partial state.
constexpr int kSliceTokens = 32;
template <typename IoT, typename CsT, int N>
__global__ void __launch_bounds__(kThreads)
chunk_state_kernel(int T, int H, int G, int L, int nc, int ks, const IoT* __restrict__ x,
                   const float* __restrict__ dt, const DtMap dtm, const float* __restrict__ A,
                   const IoT* __restrict__ Bm, CsT* __restrict__ cs, float* __restrict__ S) {
    constexpr int KT = kSliceTokens;       // tokens per smem stage
    constexpr int NT = N / 8;              // thread columns (8 n each)
    constexpr int PT = kThreads / NT;      // thread rows
    constexpr int PR = kP / PT;            // p rows per thread
    const int c = blockIdx.x / ks, sl = blockIdx.x % ks, hd = blockIdx.y, bi = blockIdx.z;
    const int g = hd / (H / G);
    const int t0 = c * L, Lc = min(L, T - t0);

    __shared__ CsT s_cs[kThreads];
    __shared__ CsT warp_tot[kThreads / 32];
    __shared__ float sX[KT][kP];
    __shared__ float sB[KT][N];
    __shared__ float sW[KT];
    // x and B of a stage are loaded into registers one stage ahead (the first before the
    // prefix sums), so their latency overlaps the scan and the previous stage's products
    constexpr int XR = KT * kP / kThreads, BR = KT * N / kThreads;
    float xr[XR], br[BR];
    auto load_stage = [&](int k0) {
        // thread column c (fixed), rows tid / W + k * (kThreads / W): one pointer step each
        {
            const int c = threadIdx.x % kP, r0 = threadIdx.x / kP;
            const IoT* src = x + (((size_t)bi * T + t0 + k0 + r0) * H + hd) * kP + c;
            const size_t step = (size_t)(kThreads / kP) * H * kP;
#pragma unroll
            for (int k = 0; k < XR; ++k, src += step)
                xr[k] = k0 + r0 + k * (kThreads / kP) < Lc ? load_io(src, 0) : 0.f;
        }
        {
            const int c = threadIdx.x % N, r0 = threadIdx.x / N;
            const IoT* src = Bm + (((size_t)bi * T + t0 + k0 + r0) * G + g) * N + c;
            const size_t step = (size_t)(kThreads / N) * G * N;
#pragma unroll
            for (int k = 0; k < BR; ++k, src += step)
                br[k] = k0 + r0 + k * (kThreads / N) < Lc ? load_io(src, 0) : 0.f;
        }
    };
    load_stage(sl * KT);
    {
        // inclusive prefix sum of a = dt*A over the chunk (tokens past its end add 0)
        const int j = threadIdx.x, lane = j & 31, w = j >> 5;
        CsT v = j < Lc ? (CsT)dt_value(dt[((size_t)bi * T + t0 + j) * H + hd], dtm, hd) * (CsT)A[hd] : CsT(0);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const CsT o = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += o;
        }
        if (lane == 31) warp_tot[w] = v;
        __syncthreads();
        for (int k = 0; k < w; ++k) v += warp_tot[k];
        s_cs[j] = v;
        if (sl == 0 && j < L) cs[(((size_t)bi * H + hd) * nc + c) * L + j] = v;
    }
    __syncthreads();
    const CsT cs_last = s_cs[Lc - 1];

    const int tn = threadIdx.x % NT, tp = threadIdx.x / NT;
    float acc[PR][8];
#pragma unroll
    for (int i = 0; i < PR; ++i)
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[i][k] = 0.f;

    for (int k0 = sl * KT; k0 < Lc; k0 += ks * KT) {
        if (threadIdx.x < KT) {
            const int t = k0 + threadIdx.x;
            sW[threadIdx.x] = t < Lc ? exp_cs(cs_last - s_cs[t]) * dt_value(dt[((size_t)bi * T + t0 + t) * H + hd], dtm, hd) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < XR; ++k) {
            const int e = threadIdx.x + k * kThreads;
            sX[e / kP][e % kP] = sW[e / kP] * xr[k];
        }
#pragma unroll
        for (int k = 0; k < BR; ++k) {
            const int e = threadIdx.x + k * kThreads;
            sB[e / N][e % N] = br[k];
        }
        __syncthreads();
        if (k0 + ks * KT < Lc) load_stage(k0 + ks * KT);
#pragma unroll 4
        for (int j = 0; j < KT; ++j) {
            float xv[PR], bv[8];
#pragma unroll
            for (int i = 0; i < PR; ++i) xv[i] = sX[j][tp * PR + i];
#pragma unroll
            for (int k = 0; k < 8; ++k) bv[k] = sB[j][tn * 8 + k];
#pragma unroll
            for (int i = 0; i < PR; ++i)
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[i][k] = fmaf(xv[i], bv[k], acc[i][k]);
        }
        __syncthreads();
    }
    float* So = S + ((((size_t)bi * nc + c) * H + hd) * ks + sl) * kP * N;
#pragma unroll
    for (int i = 0; i < PR; ++i)
#pragma unroll
        for (int k = 0; k < 8; ++k) So[(tp * PR + i) * N + tn * 8 + k] = acc[i][k];
}

// ---------------------------------------------------------------- K3
template <typename CsT, int N>
__global__ void __launch_bounds__(kThreads)
state_scan_kernel(int T, int H, int L, int nc, int ks, const CsT* __restrict__ cs,
                  const float* __restrict__ h0, float* __restrict__ S, float* __restrict__ hf) {
    const int e = blockIdx.x * kThreads + threadIdx.x;  // element of the P x N state
    const int hd = blockIdx.y, bi = blockIdx.z;
    constexpr int PN = kP * N;
    float Hs = h0 ? h0[((size_t)bi * H + hd) * PN + e] : 0.f;
    const CsT* csh = cs + ((size_t)bi * H + hd) * nc * L;
    const size_t stride = (size_t)H * ks * PN;          // from one chunk to the next
    float* Sp = S + ((size_t)bi * nc * H + hd) * ks * PN + e;
    // S_c: the slices' partial states added in slice order
    auto chunk_sum = [&](int c) {
        float v = 0.f;
        for (int sl = 0; sl < ks; ++sl) v += Sp[(size_t)c * stride + (size_t)sl * PN];
        return v;
    };
    float nxt = nc > 0 ? chunk_sum(0) : 0.f;
    for (int c = 0; c < nc; ++c) {
        const float cur = nxt;
        if (c + 1 < nc) nxt = chunk_sum(c + 1);
        const int Lc = min(L, T - c * L);
        const float gam = exp_cs(csh[(size_t)c * L + Lc - 1]);
        Sp[(size_t)c * stride] = Hs;     // H_in for chunk c (slice 0's place)
        Hs = fmaf(gam, Hs, cur);
    }
    if (hf) hf[((size_t)bi * H + hd) * PN + e] = Hs;
}

// ---------------------------------------------------------------- K4
// One CTA = TR output rows of one chunk of one (sequence, head); 16 x 16 threads, each
// RPT = TR / 16 rows x 4 columns (of p for the output, of j for a score tile).
template <typename IoT, typename CsT, int N, int TR>
__global__ void __launch_bounds__(kThreads)
chunk_output_kernel(int T, int H, int G, int L, int nc, int ks, const IoT* __restrict__ x,
                    const float* __restrict__ dt, const DtMap dtm, const IoT* __restrict__ Bm,
                    const IoT* __restrict__ Cm, const float* __restrict__ D,
                    const CsT* __restrict__ cs, const float* __restrict__ Hin,
                    IoT* __restrict__ y) {
    constexpr int TJ = 64;          // score columns j per tile
    constexpr int RPT = TR / 16;    // rows per thread
    extern __shared__ float smem[];
    float* sC = smem;               // [TR][N+1]   C rows i
    float* sK = sC + TR * (N + 1);  // [64][N+1]   H_in rows p, then B rows j
    float* sG = sK + 64 * (N + 1);  // [TR][TJ+1]  masked decayed C.B^T
    float* sX = sG + TR * (TJ + 1); // [TJ][kP]    x rows j
    __shared__ CsT s_csi[TR];
    __shared__ CsT s_csj[TJ];
    __shared__ float s_dtj[TJ];

    const int tiles_per_chunk = (L + TR - 1) / TR;
    const int c = blockIdx.x / tiles_per_chunk, it = blockIdx.x % tiles_per_chunk;
    const int hd = blockIdx.y, bi = blockIdx.z, g = hd / (H / G);
    const int t0 = c * L, Lc = min(L, T - t0), i0 = it * TR;
    if (i0 >= Lc) return;
    const CsT* csc = cs + (((size_t)bi * H + hd) * nc + c) * L;
    const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;

    auto row_ok = [&](int i) { return i < Lc; };
    const float* Hc = Hin + (((size_t)bi * nc + c) * H + hd) * ks * kP * N;
    copy_grouped<TR * N>(
        [&](int e) {
            const int i = e / N;
            return row_ok(i0 + i) ? load_io(Cm, (((size_t)bi * T + t0 + i0 + i) * G + g) * N + e % N) : 0.f;
        },
        [&](int e, float v) { sC[(e / N) * (N + 1) + e % N] = v; });
    copy_grouped<kP * N>([&](int e) { return Hc[e]; }, [&](int e, float v) { sK[(e / N) * (N + 1) + e % N] = v; });
    if (threadIdx.x < TR) s_csi[threadIdx.x] = row_ok(i0 + threadIdx.x) ? csc[i0 + threadIdx.x] : CsT(0);
    __syncthreads();

    // state-to-output term: Y[i][p] = exp(cs_i) * sum_n C[i][n] H[p][n]
    float acc[RPT][4];
#pragma unroll
    for (int a = 0; a < RPT; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
    for (int n = 0; n < N; ++n) {
        float cv[RPT], hv[4];
#pragma unroll
        for (int a = 0; a < RPT; ++a) cv[a] = sC[(tr * RPT + a) * (N + 1) + n];
#pragma unroll
        for (int q = 0; q < 4; ++q) hv[q] = sK[(tc * 4 + q) * (N + 1) + n];
#pragma unroll
        for (int a = 0; a < RPT; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[a][q] = fmaf(cv[a], hv[q], acc[a][q]);
    }
#pragma unroll
    for (int a = 0; a < RPT; ++a) {
        const float e = exp_cs(s_csi[tr * RPT + a]);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][q] *= e;
    }

    // intra-chunk dual form over column tiles j0 <= i0 + TR - 1
    for (int j0 = 0; j0 < i0 + TR && j0 < Lc; j0 += TJ) {
        __syncthreads();
        copy_grouped<TJ * N>(
            [&](int e) {
                const int j = e / N;
                return (j0 + j < Lc) ? load_io(Bm, (((size_t)bi * T + t0 + j0 + j) * G + g) * N + e % N) : 0.f;
            },
            [&](int e, float v) { sK[(e / N) * (N + 1) + e % N] = v; });
        copy_grouped<TJ * kP>(
            [&](int e) {
                const int j = e / kP;
                return (j0 + j < Lc) ? load_io(x, (((size_t)bi * T + t0 + j0 + j) * H + hd) * kP + e % kP) : 0.f;
            },
            [&](int e, float v) { sX[e] = v; });
        if (threadIdx.x < TJ) {
            const int j = j0 + threadIdx.x;
            s_csj[threadIdx.x] = j < Lc ? csc[j] : CsT(0);
            s_dtj[threadIdx.x] = j < Lc ? dt_value(dt[((size_t)bi * T + t0 + j) * H + hd], dtm, hd) : 0.f;
        }
        __syncthreads();
        // G = C_i . B_j over this TR x 64 tile
        float gacc[RPT][4];
#pragma unroll
        for (int a = 0; a < RPT; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) gacc[a][q] = 0.f;
        for (int n = 0; n < N; ++n) {
            float cv[RPT], bv[4];
#pragma unroll
            for (int a = 0; a < RPT; ++a) cv[a] = sC[(tr * RPT + a) * (N + 1) + n];
#pragma unroll
            for (int q = 0; q < 4; ++q) bv[q] = sK[(tc * 4 + q) * (N + 1) + n];
#pragma unroll
            for (int a = 0; a < RPT; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) gacc[a][q] = fmaf(cv[a], bv[q], gacc[a][q]);
        }
        // decay, causal mask and dt_j; the mask is a fixed function of (i, j)
#pragma unroll
        for (int a = 0; a < RPT; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int il = tr * RPT + a, jl = tc * 4 + q;
                float v = 0.f;
                if (j0 + jl <= i0 + il)
                    v = gacc[a][q] * exp_cs(s_csi[il] - s_csj[jl]) * s_dtj[jl];
                sG[il * (TJ + 1) + jl] = v;
            }
        __syncthreads();
        for (int j = 0; j < TJ; ++j) {
            float gv[RPT], xv[4];
#pragma unroll
            for (int a = 0; a < RPT; ++a) gv[a] = sG[(tr * RPT + a) * (TJ + 1) + j];
#pragma unroll
            for (int q = 0; q < 4; ++q) xv[q] = sX[j * kP + tc * 4 + q];
#pragma unroll
            for (int a = 0; a < RPT; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[a][q] = fmaf(gv[a], xv[q], acc[a][q]);
        }
    }
    const float Dv = D[hd];
#pragma unroll
    for (int a = 0; a < RPT; ++a) {
        const int i = i0 + tr * RPT + a;
        if (i >= Lc) continue;
        const size_t off = (((size_t)bi * T + t0 + i) * H + hd) * kP;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int p = tc * 4 + q;
            store_io(y, off + p, acc[a][q] + Dv * load_io(x, off + p));
        }
    }
}

// K4 for grids too small to fill the GPU: one CTA = 16 output rows of one chunk of one
// (sequence, head).  The CTAs of rows late in a chunk see up to four 64-column tiles and set
// the kernel's length, so each product is register-blocked to shorten their serial chain: a
// thread owns a 4 x 4 block of its output and one quarter of the contraction (kq =
// threadIdx.x / 64), and one step reads two 16-byte shared values (four rows of one operand,
// four columns of the other) for sixteen FMAs.  The quarters are added in order through
// shared memory: the scores after every column tile, y once at the end.  C, B and H_in are
// kept transposed ([n][i], [n][j], [n][p]), the masked decayed scores transposed ([j][i]),
// x row-major.  All copies are asynchronous into a ring of kDepth column tiles (the whole
// 256-token chunk at N = 64), so up to kDepth - 1 tiles are in flight while one is evaluated.
constexpr int kSmallRows = 16, kSmallCols = 64;
constexpr int kLdT = 68, kLdR = 20;  // rows of 64 and of 16 floats, padded to keep 16-byte alignment
constexpr int kSplit = kThreads / ((kSmallRows / 4) * (kSmallCols / 4));  // contraction quarters
template <int N>
constexpr int small_depth() { return N == 64 ? 4 : 2; }
template <int N>
constexpr size_t small_smem_bytes() {
    return sizeof(float) * (N * kLdR + N * kLdT + small_depth<N>() * (N * kLdT + kSmallCols * kP) +
                            kSplit * kSmallRows * kLdT + kSmallCols * kLdR);
}

// a[r][q] += u[r] * v[q]
__device__ __forceinline__ void fma_4x4(float (&a)[4][4], const float4 u, const float4 v) {
    const float ur[4] = {u.x, u.y, u.z, u.w}, vq[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) a[r][q] = fmaf(ur[r], vq[q], a[r][q]);
}

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }

template <typename IoT, typename CsT, int N>
__global__ void __launch_bounds__(kThreads)
chunk_output_small_kernel(int T, int H, int G, int L, int nc, int ks, const IoT* __restrict__ x,
                          const float* __restrict__ dt, const DtMap dtm, const IoT* __restrict__ Bm,
                          const IoT* __restrict__ Cm, const float* __restrict__ D,
                          const CsT* __restrict__ cs, const float* __restrict__ Hin,
                          IoT* __restrict__ y) {
    constexpr int TR = kSmallRows, TJ = kSmallCols, kDepth = small_depth<N>();
    constexpr int NQ = N / kSplit, JQ = TJ / kSplit;  // contraction length of one quarter
    static_assert(TJ == kP && kSplit == 4 && TR * TJ == 4 * kThreads, "4 x 4 blocks, four quarters");
    extern __shared__ __align__(16) float smem[];
    float* sCT = smem;                     // [N][kLdR]            C, transposed: [n][i]
    float* sHT = sCT + N * kLdR;           // [N][kLdT]            H_in, transposed: [n][p]
    float* sBT = sHT + N * kLdT;           // [kDepth][N][kLdT]    B, transposed: [n][j]
    float* sX = sBT + kDepth * N * kLdT;   // [kDepth][TJ][kP]     x rows j
    float* sQ = sX + kDepth * TJ * kP;     // [kSplit][TR][kLdT]   quarter partials: scores, then y
    float* sGT = sQ + kSplit * TR * kLdT;  // [TJ][kLdR]           masked decayed scores, transposed: [j][i]
    __shared__ CsT s_csi[TR];
    __shared__ CsT s_csj[kDepth][TJ];
    __shared__ float s_dtj[kDepth][TJ];

    const int tiles_per_chunk = (L + TR - 1) / TR;
    const int c = blockIdx.x / tiles_per_chunk, it = blockIdx.x % tiles_per_chunk;
    const int hd = blockIdx.y, bi = blockIdx.z, g = hd / (H / G);
    const int t0 = c * L, Lc = min(L, T - t0), i0 = it * TR;
    if (i0 >= Lc) return;
    const int ntile = (min(i0 + TR, Lc) + TJ - 1) / TJ;  // column tiles at and below the diagonal
    const CsT* csc = cs + (((size_t)bi * H + hd) * nc + c) * L;
    // quarter kq of the contraction; output rows 4 ri .. 4 ri + 3, columns 4 ci .. 4 ci + 3
    const int kq = threadIdx.x / 64, ri = (threadIdx.x % 64) / 16, ci = threadIdx.x % 16;

    auto issue_tile = [&](int t) {  // B, x, dt and the prefix sums of column tile t into slot t % kDepth
        if (t >= ntile) return;
        const int j0 = t * TJ, buf = t % kDepth;
        tile_load<N, TJ, true>(sBT + buf * N * kLdT, kLdT, Bm + (((size_t)bi * T + t0 + j0) * G + g) * N,
                               (size_t)G * N, Lc - j0);
        tile_load<kP, TJ, false>(sX + buf * TJ * kP, kP, x + (((size_t)bi * T + t0 + j0) * H + hd) * kP,
                                 (size_t)H * kP, Lc - j0);
        if (threadIdx.x < TJ) {
            const int j = j0 + threadIdx.x;
            s_dtj[buf][threadIdx.x] = j < Lc ? dt_value(dt[((size_t)bi * T + t0 + j) * H + hd], dtm, hd) : 0.f;
            s_csj[buf][threadIdx.x] = j < Lc ? csc[j] : CsT(0);
        }
    };

    // copy groups, oldest first: {C, tile 0}, {H_in}, {tile 1} .. {tile kDepth - 1}, then one
    // per loop iteration (empty where there is no tile), so that tile t is complete once at
    // most kDepth - 1 groups are pending
    tile_load<N, TR, true>(sCT, kLdR, Cm + (((size_t)bi * T + t0 + i0) * G + g) * N, (size_t)G * N, Lc - i0);
    issue_tile(0);
    cp_async_commit();
    const float* Hc = Hin + (((size_t)bi * nc + c) * H + hd) * ks * kP * N;
    tile_load<N, kP, true>(sHT, kLdT, Hc, (size_t)N, kP);
    cp_async_commit();
#pragma unroll
    for (int t = 1; t < kDepth; ++t) {
        issue_tile(t);
        cp_async_commit();
    }
    if (threadIdx.x < TR) s_csi[threadIdx.x] = i0 + threadIdx.x < Lc ? csc[i0 + threadIdx.x] : CsT(0);
    cp_async_wait<kDepth - 1>();  // C, tile 0 and H_in landed
    __syncthreads();

    const float* cq = sCT + kq * NQ * kLdR + 4 * ri;  // this thread's C rows, from its quarter's first n
    // state-to-output term, this quarter of n: Y[i][p] = exp(cs_i) * sum_n C[i][n] H[p][n]
    float acc[4][4] = {};
    {
        const float* hq = sHT + kq * NQ * kLdT + 4 * ci;
#pragma unroll 4
        for (int n = 0; n < NQ; ++n) fma_4x4(acc, lds4(cq + n * kLdR), lds4(hq + n * kLdT));
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float e = exp_cs(s_csi[4 * ri + r]);
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[r][q] *= e;
        }
    }

    // intra-chunk dual form over the column tiles
#pragma unroll 1
    for (int t = 0; t < ntile; ++t) {
        const int j0 = t * TJ, buf = t % kDepth;
        if (t > 0) {
            cp_async_wait<kDepth - 1>();  // tile t landed
            __syncthreads();
        }
        {   // scores, this quarter of n: S[i][j] = sum_n C[i][n] B[j][n]
            const float* bq = sBT + buf * N * kLdT + kq * NQ * kLdT + 4 * ci;
            float sc[4][4] = {};
#pragma unroll 4
            for (int n = 0; n < NQ; ++n) fma_4x4(sc, lds4(cq + n * kLdR), lds4(bq + n * kLdT));
#pragma unroll
            for (int r = 0; r < 4; ++r)
                *reinterpret_cast<float4*>(sQ + (kq * TR + 4 * ri + r) * kLdT + 4 * ci) =
                    make_float4(sc[r][0], sc[r][1], sc[r][2], sc[r][3]);
        }
        __syncthreads();
        {   // the quarters added in order, then the decay and the causal mask: thread (column
            // jl, rows 4 r4 .. 4 r4 + 3) writes one 16-byte row of the transposed scores
            const int jl = threadIdx.x % TJ, r4 = threadIdx.x / TJ;
            float v[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = 4 * r4 + r;
                float sv = sQ[i * kLdT + jl];
#pragma unroll
                for (int q = 1; q < kSplit; ++q) sv += sQ[(q * TR + i) * kLdT + jl];
                v[r] = j0 + jl <= i0 + i ? sv * exp_cs(s_csi[i] - s_csj[buf][jl]) * s_dtj[buf][jl] : 0.f;
            }
            *reinterpret_cast<float4*>(sGT + jl * kLdR + 4 * r4) = make_float4(v[0], v[1], v[2], v[3]);
        }
        __syncthreads();
        // this quarter of the tile's columns: Y[i][p] += sum_j S~[i][j] x[j][p]; a quarter wholly
        // above the diagonal adds nothing (kq is the same across a warp)
        if (j0 + kq * JQ <= i0 + TR - 1) {
            const float* gq = sGT + kq * JQ * kLdR + 4 * ri;
            const float* xq = sX + buf * TJ * kP + kq * JQ * kP + 4 * ci;
#pragma unroll 4
            for (int j = 0; j < JQ; ++j) fma_4x4(acc, lds4(gq + j * kLdR), lds4(xq + j * kP));
        }
        __syncthreads();  // slot t % kDepth, the partials and the scores are free
        issue_tile(t + kDepth);
        cp_async_commit();
    }

    // the quarters of y added in order, then the D skip: thread (row, columns 4 pc .. 4 pc + 3)
#pragma unroll
    for (int r = 0; r < 4; ++r)
        *reinterpret_cast<float4*>(sQ + (kq * TR + 4 * ri + r) * kLdT + 4 * ci) =
            make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    __syncthreads();
    const int row = threadIdx.x / 16, pc = threadIdx.x % 16;
    const int i = i0 + row;
    if (i < Lc) {
        float4 sv = lds4(sQ + row * kLdT + 4 * pc);
#pragma unroll
        for (int q = 1; q < kSplit; ++q) {
            const float4 u = lds4(sQ + (q * TR + row) * kLdT + 4 * pc);
            sv.x += u.x;
            sv.y += u.y;
            sv.z += u.z;
            sv.w += u.w;
        }
        const float out[4] = {sv.x, sv.y, sv.z, sv.w};
        const float Dv = D[hd];
        const size_t off = (((size_t)bi * T + t0 + i) * H + hd) * kP;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int p = 4 * pc + q;
            store_io(y, off + p, out[q] + Dv * load_io(x, off + p));
        }
    }
}

// SMs of the device current at the first call (148 when no device answers); initialised
// once, thread-safely
int sm_count_simt() {
    static const int n = [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            v <= 0)
            v = 148;
        return v;
    }();
    return n;
}

// Slices per chunk for the chunk-state pass: enough CTAs for two per SM when (chunks x
// heads x sequences) alone fall short, at most one per 32 tokens of the chunk, and at most
// 256 MB of partial states.
int state_slices(int b, int T, int H, int N, int L) {
    const int nc = (T + L - 1) / L;
    const double units = (double)nc * H * b;
    int ks = (int)std::ceil(2.0 * sm_count_simt() / std::max(units, 1.0));
    ks = std::max(1, std::min(ks, L / kSliceTokens));
    while (ks > 1 && units * ks * kP * N * sizeof(float) > 256.0 * 1024 * 1024) --ks;
    return ks;
}

// K4: 64-row tiles, or the pipelined, register-blocked 16-row kernel when 64-row tiles would
// not give every SM two CTAs
template <typename IoT, typename CsT, int N>
int launch_output(int b, int T, int H, int G, int L, int nc, int ks, const IoT* x, const float* dt, const DtMap& dtm,
                  const IoT* Bm, const IoT* Cm, const float* D, const CsT* cs, const float* S, void* y, cudaStream_t s) {
    const bool small = (double)nc * ((L + 63) / 64) * H * b < 2.0 * sm_count_simt();
    const int TR = small ? kSmallRows : 64;
    const size_t smem = small ? small_smem_bytes<N>() : sizeof(float) * (64 * (N + 1) + 64 * (N + 1) + 64 * 65 + 64 * kP);
    auto k4 = small ? chunk_output_small_kernel<IoT, CsT, N> : chunk_output_kernel<IoT, CsT, N, 64>;
    if (const int st = smem_limit_once((const void*)k4, (int)smem)) return st;
    LaunchScope ls("simt_chunk_output", s);
    k4<<<dim3(nc * ((L + TR - 1) / TR), H, b), kThreads, smem, s>>>(T, H, G, L, nc, ks, x, dt, dtm, Bm, Cm, D, cs, S,
                                                                     static_cast<IoT*>(y));
    return SSD_OK;
}

template <typename IoT, typename CsT, int N>
int run(int b, int T, int H, int G, int L, const void* x, const float* dt, const DtMap dtm, const float* A,
        const void* Bm, const void* Cm, const float* D, const float* h0, void* y, float* hf,
        char* ws, cudaStream_t s) {
    const int nc = (T + L - 1) / L;
    const int ks = state_slices(b, T, H, N, L);
    CsT* cs = reinterpret_cast<CsT*>(ws);
    float* S = reinterpret_cast<float*>(ws + round_up((size_t)b * H * nc * L * sizeof(CsT), 256));
    const IoT* xi = static_cast<const IoT*>(x);
    const IoT* Bi = static_cast<const IoT*>(Bm);
    const IoT* Ci = static_cast<const IoT*>(Cm);
    if (const int st = smem_limit_once((const void*)chunk_state_kernel<IoT, CsT, N>, 0)) return st;
    if (const int st = smem_limit_once((const void*)state_scan_kernel<CsT, N>, 0)) return st;
    {
        LaunchScope ls("simt_chunk_state", s);
        chunk_state_kernel<IoT, CsT, N><<<dim3(nc * ks, H, b), kThreads, 0, s>>>(T, H, G, L, nc, ks, xi, dt, dtm, A, Bi,
                                                                                  cs, S);
    }
    {
        LaunchScope ls("simt_state_scan", s);
        state_scan_kernel<CsT, N><<<dim3(kP * N / kThreads, H, b), kThreads, 0, s>>>(T, H, L, nc, ks, cs, h0, S, hf);
    }
    const int st = launch_output<IoT, CsT, N>(b, T, H, G, L, nc, ks, xi, dt, dtm, Bi, Ci, D, cs, S, y, s);
    if (st != SSD_OK) return st;
    SSD_CUDA_TRY(cudaGetLastError());
    return SSD_OK;
}

}  // namespace

size_t prefill_simt_workspace_bytes(int b, int T, int H, int N, int L, int io) {
    const int nc = (T + L - 1) / L;
    const size_t cs_elem = io == SSD_F32 ? sizeof(double) : sizeof(float);
    return round_up((size_t)b * H * nc * L * cs_elem, 256) +
           round_up((size_t)b * nc * H * state_slices(b, T, H, N, L) * kP * N * sizeof(float), 256);
}

int launch_prefill_simt(int b, int T, int H, int N, int G, int L, int io, const void* x,
                        const float* dt, const DtMap& dtm, const float* A, const void* Bm, const void* Cm,
                        const float* D, const float* h0, void* y, float* hf, void* ws,
                        cudaStream_t s) {
    char* w = static_cast<char*>(ws);
    if (io == SSD_F32) {
        return N == 128 ? run<float, double, 128>(b, T, H, G, L, x, dt, dtm, A, Bm, Cm, D, h0, y, hf, w, s)
                        : run<float, double, 64>(b, T, H, G, L, x, dt, dtm, A, Bm, Cm, D, h0, y, hf, w, s);
    }
    return N == 128 ? run<__nv_bfloat16, float, 128>(b, T, H, G, L, x, dt, dtm, A, Bm, Cm, D, h0, y, hf, w, s)
                    : run<__nv_bfloat16, float, 64>(b, T, H, G, L, x, dt, dtm, A, Bm, Cm, D, h0, y, hf, w, s);
}

}  // namespace ssd
