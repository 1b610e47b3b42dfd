// decode.cu -- the O(1) cached decode step and its on-device loop (CUDA graph).
//
// Method: "Compiler-First State Space Duality and Portable O(1) Autoregressive Caching"
// (arXiv 2603.09555), O(1) caching section: a depthwise convolution over a sliding window
// of k-1 cached inputs, then one recurrence step h_t = Abar h_{t-1} + Bbar x_t with
// Abar = exp(dt*A) (scalar per head) and Bbar x = dt * x B^T; y = h C + D x.  The
// "Compiled on-device loops" paragraph motivates running many steps with no host
// round trip, done here with one CUDA graph of dependent step kernels.
//
// Bound: HBM.  Every step must stream the whole fp32 SSM state (layers*b*H*P*N*4 bytes)
// in and out; everything else (conv state, inputs, weights, y) is a few percent of that.
// One CTA owns one (layer, sequence, head): it reads its P x N state once with 16-byte
// loads issued back to back, applies the update, reduces y over N with warp shuffles and
// writes the state back.  The B/C conv channels are shared by the H/G heads of a group:
// every head CTA recomputes them from the old window, and the last CTA of the group to
// finish (an arrival counter, no waiting) writes the shifted window back.
#include "common.cuh"

#include <cuda.h>

#include <mutex>
#include <vector>

namespace ssd {

namespace {

constexpr int kDecodeThreads = 256;
constexpr int kP = 64;

template <typename IoT, int N, int ACT>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_kernel(int layers, int b, int H, int G, float* __restrict__ h,
                   float* __restrict__ conv_state, const IoT* __restrict__ xbc,
                   const float* __restrict__ dt, const float* __restrict__ A,
                   const float* __restrict__ D, const float* __restrict__ conv_w,
                   const float* __restrict__ conv_b, IoT* __restrict__ y,
                   unsigned int* __restrict__ arrivals) {
    constexpr int K = 4, KM1 = 3;
    constexpr int VEC_PER_ROW = N / 4;                    // float4 per state row
    constexpr int ROWS_PER_PASS = kDecodeThreads / VEC_PER_ROW;
    constexpr int PASSES = kP / ROWS_PER_PASS;            // 8 (N=128) or 4 (N=64)
    static_assert(kP % ROWS_PER_PASS == 0, "rows");

    const int hd = blockIdx.x, r = blockIdx.y, l = blockIdx.z;
    const int hpg = H / G, g = hd / hpg;
    const int Dc = H * kP + 2 * G * N;
    const int tid = threadIdx.x;
    const size_t lr = (size_t)l * b + r;

    __shared__ float s_x[kP];
    __shared__ __align__(16) float s_B[N];
    __shared__ __align__(16) float s_C[N];
    __shared__ int s_last;

    // ---- issue the state loads first: they are the bandwidth that matters
    const size_t hbase = ((lr * H + hd) * kP) * N;
    float4* hv = reinterpret_cast<float4*>(h + hbase);
    float4 st[PASSES];
    const int vcol = tid % VEC_PER_ROW, vrow = tid / VEC_PER_ROW;
#pragma unroll
    for (int i = 0; i < PASSES; ++i) st[i] = hv[(size_t)(vrow + i * ROWS_PER_PASS) * VEC_PER_ROW + vcol];

    // ---- conv: x channels of this head (owned: window written back here)
    //      B/C channels of group g (shared: window written back by the last head CTA)
    const float* cw = conv_w + (size_t)l * Dc * K;
    const float* cb = conv_b + (size_t)l * Dc;
    float* cst = conv_state + lr * Dc * KM1;
    const IoT* xin = xbc + lr * Dc;
    float keep0 = 0.f, keep1 = 0.f, keep2 = 0.f;  // window[1..3] of a B/C channel
    int bc_chan = -1;
    if (tid < kP) {
        const int c = hd * kP + tid;
        const float w0 = cw[c * K + 0], w1 = cw[c * K + 1], w2 = cw[c * K + 2], w3 = cw[c * K + 3];
        const float s0 = cst[c * KM1 + 0], s1 = cst[c * KM1 + 1], s2 = cst[c * KM1 + 2];
        const float xi = load_io(xin, c);
        float u = cb[c] + w0 * s0 + w1 * s1 + w2 * s2 + w3 * xi;
        if (ACT == SSD_ACT_SILU) u = u / (1.f + __expf(-u));
        s_x[tid] = u;
        cst[c * KM1 + 0] = s1;
        cst[c * KM1 + 1] = s2;
        cst[c * KM1 + 2] = xi;
    }
    for (int j = tid; j < 2 * N; j += kDecodeThreads) {
        const int c = H * kP + (j < N ? g * N + j : G * N + g * N + (j - N));
        const float w0 = cw[c * K + 0], w1 = cw[c * K + 1], w2 = cw[c * K + 2], w3 = cw[c * K + 3];
        const float s0 = cst[c * KM1 + 0], s1 = cst[c * KM1 + 1], s2 = cst[c * KM1 + 2];
        const float xi = load_io(xin, c);
        float u = cb[c] + w0 * s0 + w1 * s1 + w2 * s2 + w3 * xi;
        if (ACT == SSD_ACT_SILU) u = u / (1.f + __expf(-u));
        if (j < N) s_B[j] = u; else s_C[j - N] = u;
        bc_chan = c; keep0 = s1; keep1 = s2; keep2 = xi;
    }
    __syncthreads();

    // ---- arrival: every read of the shared B/C window above is complete (its values
    //      are in s_B/s_C); the last head CTA of the group writes the shifted window.
    if (tid == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(&arrivals[lr * G + g], 1u);
        s_last = (prev == (unsigned int)(hpg - 1));
        if (s_last) arrivals[lr * G + g] = 0u;  // ready for the next step (stream-ordered)
    }

    // ---- SSM step on the state rows this thread holds
    const float dtv = dt[lr * H + hd];
    const float alpha = __expf(dtv * A[(size_t)l * H + hd]);
    const float Dv = D[(size_t)l * H + hd];
    const float4 bv = reinterpret_cast<const float4*>(s_B)[vcol];
    const float4 cv = reinterpret_cast<const float4*>(s_C)[vcol];
    float part[PASSES];
#pragma unroll
    for (int i = 0; i < PASSES; ++i) {
        const int p = vrow + i * ROWS_PER_PASS;
        const float dx = dtv * s_x[p];
        float4 v = st[i];
        v.x = fmaf(alpha, v.x, dx * bv.x);
        v.y = fmaf(alpha, v.y, dx * bv.y);
        v.z = fmaf(alpha, v.z, dx * bv.z);
        v.w = fmaf(alpha, v.w, dx * bv.w);
        hv[(size_t)p * VEC_PER_ROW + vcol] = v;
        part[i] = v.x * cv.x + v.y * cv.y + v.z * cv.z + v.w * cv.w;
    }
    // reduce each row over its VEC_PER_ROW lanes (32 for N=128, 16 for N=64)
#pragma unroll
    for (int i = 0; i < PASSES; ++i) {
#pragma unroll
        for (int off = VEC_PER_ROW / 2; off > 0; off >>= 1)
            part[i] += __shfl_xor_sync(0xffffffffu, part[i], off);
    }
    if (vcol == 0) {
        IoT* yo = y + (lr * H + hd) * kP;
#pragma unroll
        for (int i = 0; i < PASSES; ++i) {
            const int p = vrow + i * ROWS_PER_PASS;
            store_io(yo, p, part[i] + Dv * s_x[p]);
        }
    }

    __syncthreads();
    if (s_last && bc_chan >= 0) {
        cst[bc_chan * KM1 + 0] = keep0;
        cst[bc_chan * KM1 + 1] = keep1;
        cst[bc_chan * KM1 + 2] = keep2;
    }
}

typedef void (*decode_fn)(int, int, int, int, float*, float*, const void*, const float*,
                          const float*, const float*, const float*, const float*, void*,
                          unsigned int*);

template <typename IoT, int N, int ACT>
void* kernel_ptr() {
    return reinterpret_cast<void*>(&decode_step_kernel<IoT, N, ACT>);
}

void* pick_kernel(int io, int N, int act) {
    if (io == SSD_BF16) {
        if (N == 128) return act ? kernel_ptr<__nv_bfloat16, 128, 1>() : kernel_ptr<__nv_bfloat16, 128, 0>();
        return act ? kernel_ptr<__nv_bfloat16, 64, 1>() : kernel_ptr<__nv_bfloat16, 64, 0>();
    }
    if (N == 128) return act ? kernel_ptr<float, 128, 1>() : kernel_ptr<float, 128, 0>();
    return act ? kernel_ptr<float, 64, 1>() : kernel_ptr<float, 64, 0>();
}

}  // namespace

size_t decode_workspace_bytes(int layers, int b, int G) {
    return round_up((size_t)layers * b * G * sizeof(unsigned int), 256);
}

// Argument pack for one step kernel (kept alive for graph-node creation).
struct StepArgs {
    int layers, b, H, G;
    float* h;
    float* conv_state;
    const void* xbc;
    const float* dt;
    const float* A;
    const float* D;
    const float* conv_w;
    const float* conv_b;
    void* y;
    unsigned int* arrivals;
    void* params[14];
    void fill() {
        params[0] = &layers; params[1] = &b; params[2] = &H; params[3] = &G;
        params[4] = &h; params[5] = &conv_state; params[6] = &xbc; params[7] = &dt;
        params[8] = &A; params[9] = &D; params[10] = &conv_w; params[11] = &conv_b;
        params[12] = &y; params[13] = &arrivals;
    }
};

int launch_decode_step(int layers, int b, int H, int N, int G, int act, int io, float* h,
                       float* conv_state, const void* xbc, const float* dt, const float* A,
                       const float* D, const float* conv_w, const float* conv_b, void* y,
                       void* ws, cudaStream_t s) {
    SSD_CUDA_TRY(cudaMemsetAsync(ws, 0, (size_t)layers * b * G * sizeof(unsigned int), s));
    StepArgs a{layers, b, H, G, h, conv_state, xbc, dt, A, D, conv_w, conv_b, y,
               reinterpret_cast<unsigned int*>(ws)};
    a.fill();
    dim3 grid(H, b, layers);
    {
        LaunchScope ls("decode_step", s);
        SSD_CUDA_TRY(cudaLaunchKernel(pick_kernel(io, N, act), grid, dim3(kDecodeThreads), a.params, 0, s));
    }
    return SSD_OK;
}

}  // namespace ssd

// ---------------------------------------------------------------------------------------
// Decode plan: one CUDA graph = counter reset + n_steps dependent step kernels.
struct ssd_decode_plan {
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    int n_steps = 0;
};

namespace ssd {

int create_decode_plan(ssd_decode_plan** out, int layers, int b, int H, int N, int G, int act,
                       int io, float* h, float* conv_state, const void* xbc_ring,
                       const float* dt_ring, int ring, const float* A, const float* D,
                       const float* conv_w, const float* conv_b, void* y_ring, int n_steps,
                       void* ws) {
    const int P = kP;
    const size_t Dc = (size_t)H * P + 2 * (size_t)G * N;
    const size_t io_bytes = io == SSD_BF16 ? 2 : 4;
    const size_t xbc_step = (size_t)layers * b * Dc * io_bytes;
    const size_t dt_step = (size_t)layers * b * H;
    const size_t y_step = (size_t)layers * b * H * P * io_bytes;

    ssd_decode_plan* plan = new ssd_decode_plan();
    plan->n_steps = n_steps;
    cudaError_t e = cudaGraphCreate(&plan->graph, 0);
    if (e != cudaSuccess) { delete plan; return cuda_status(e, "cudaGraphCreate"); }

    cudaGraphNode_t prev = nullptr;
    cudaMemsetParams mp{};
    mp.dst = ws;
    mp.value = 0;
    mp.elementSize = 4;
    mp.width = (size_t)layers * b * G;
    mp.height = 1;
    mp.pitch = 0;
    e = cudaGraphAddMemsetNode(&prev, plan->graph, nullptr, 0, &mp);
    void* fn = pick_kernel(io, N, act);
    std::vector<StepArgs> args(n_steps > 0 ? 1 : 0);
    for (int t = 0; e == cudaSuccess && t < n_steps; ++t) {
        const int slot = t % ring;
        StepArgs a{layers, b, H, G, h, conv_state,
                   static_cast<const char*>(xbc_ring) + slot * xbc_step,
                   dt_ring + slot * dt_step, A, D, conv_w, conv_b,
                   static_cast<char*>(y_ring) + slot * y_step,
                   reinterpret_cast<unsigned int*>(ws)};
        a.fill();
        cudaKernelNodeParams kp{};
        kp.func = fn;
        kp.gridDim = dim3(H, b, layers);
        kp.blockDim = dim3(kDecodeThreads);
        kp.sharedMemBytes = 0;
        kp.kernelParams = a.params;  // values are copied into the node here
        cudaGraphNode_t node;
        e = cudaGraphAddKernelNode(&node, plan->graph, &prev, 1, &kp);
        prev = node;
    }
    if (e == cudaSuccess) e = cudaGraphInstantiate(&plan->exec, plan->graph, 0);
    if (e != cudaSuccess) {
        if (plan->graph) cudaGraphDestroy(plan->graph);
        delete plan;
        return cuda_status(e, "decode plan graph build");
    }
    *out = plan;
    return SSD_OK;
}

int launch_decode_plan(ssd_decode_plan* plan, cudaStream_t s) {
    LaunchScope ls("decode_plan", s, (uint64_t)plan->n_steps);
    SSD_CUDA_TRY(cudaGraphLaunch(plan->exec, s));
    return SSD_OK;
}

int destroy_decode_plan(ssd_decode_plan* plan) {
    cudaError_t e1 = plan->exec ? cudaGraphExecDestroy(plan->exec) : cudaSuccess;
    cudaError_t e2 = plan->graph ? cudaGraphDestroy(plan->graph) : cudaSuccess;
    delete plan;
    if (e1 != cudaSuccess) return cuda_status(e1, "cudaGraphExecDestroy");
    if (e2 != cudaSuccess) return cuda_status(e2, "cudaGraphDestroy");
    return SSD_OK;
}

}  // namespace ssd

// ---------------------------------------------------------------------------------------
// Scratch for the allocation-free decode step: the arrival counters live in a file-scope
// device array instead of a caller workspace.  Every GPU that loads the library holds it
// (SSD_DECODE_NOALLOC_MAX_COUNTERS x 4 bytes) until the process exits.  In host code the
// name g_noalloc_arrivals is only a stand-in; its device address is looked up per device.
static __device__ __align__(256) unsigned int g_noalloc_arrivals[SSD_DECODE_NOALLOC_MAX_COUNTERS];

namespace ssd {

// Device address and size of the scratch array in the current context.  The address is
// looked up (cudaGetSymbolAddress) the first time a context calls, with that context
// current, and cached under the context's unique id: a context created later on the same
// device -- after cudaDeviceReset, or a caller's own non-primary context -- has a new id
// and gets its own lookup, so no call ever uses an address from a context that is gone.
namespace {
using PFN_ctxGetCurrent = CUresult (*)(CUcontext*);
using PFN_ctxGetId = CUresult (*)(CUcontext, unsigned long long*);
template <typename F>
F driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<F>(p);
}
// unique id of the current context (0 if none is current or the driver cannot say)
unsigned long long current_context_id() {
    static PFN_ctxGetCurrent get_cur = driver_fn<PFN_ctxGetCurrent>("cuCtxGetCurrent");
    static PFN_ctxGetId get_id = driver_fn<PFN_ctxGetId>("cuCtxGetId");
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}
}  // namespace

int decode_noalloc_scratch(void** ptr, size_t* bytes) {
    constexpr int kSlots = 64;
    static std::mutex mu;
    static unsigned long long ids[kSlots] = {};
    static void* addrs[kSlots] = {};
    static int next = 0;
    // the lookup also makes the device's primary context current if nothing is yet
    void* p = nullptr;
    unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(mu);
    if (id != 0)
        for (int i = 0; i < kSlots; ++i)
            if (ids[i] == id) {
                *ptr = addrs[i];
                *bytes = sizeof(g_noalloc_arrivals);
                return SSD_OK;
            }
    SSD_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_arrivals));
    if (id == 0) id = current_context_id();  // the lookup created the primary context
    if (id != 0) {
        ids[next] = id;
        addrs[next] = p;
        next = (next + 1) % kSlots;
    }
    *ptr = p;
    *bytes = sizeof(g_noalloc_arrivals);
    return SSD_OK;
}

}  // namespace ssd
