// api.cu -- the extern "C" boundary of libssd_b200.so (declared in include/ssd.h).
//
// Host-side only: argument validation (before anything is enqueued), workspace carving
// and dispatch to the sm_100a kernels.  No device memory is allocated here.
#include "common.cuh"

#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

namespace ssd {

// kernels (defined in the other translation units)
size_t prefill_simt_workspace_bytes(int b, int T, int H, int N, int L, int io);
int launch_prefill_simt(int b, int T, int H, int N, int G, int L, int io, const void* x,
                        const float* dt, const DtMap& dtm, const float* A, const void* Bm, const void* Cm,
                        const float* D, const float* h0, void* y, float* hf, void* ws,
                        cudaStream_t s);
bool prefill_tc_supported(int P, int N, int io);
size_t prefill_tc_workspace_bytes(int b, int T, int H);
int launch_prefill_tc(int b, int T, int H, int G, const void* x, const float* dt, const DtMap& dtm, const float* A,
                      const void* Bm,
                      const void* Cm, const float* D, const float* h0, void* y, float* hf, void* ws,
                      cudaStream_t s);
int prefill_tc_status(void* ws, cudaStream_t s);
void prefill_tc_starve_next(unsigned long long wait_ns);
void prefill_tc_force_segments(int nseg);
void prefill_tc_force_split(int n_full, int nseg);
void prefill_tc_decay_mode(int mode);
int prefill_tc_segments(int b, int T, int H);
int prefill_tc_whole_units(int b, int T, int H);
size_t prefill_tc_local_state_workspace_bytes(int b, int T, int H);
int launch_prefill_tc_local_state(int b, int T, int H, int G, const void* x, const float* dt, const float* A,
                                  const void* Bm, float* h_local, float* log_decay, void* ws, cudaStream_t s);
int launch_context_scan(int rank, int b, int H, const float* h0, const float* h_all, const float* ld_all,
                        float* h_in, cudaStream_t s);
size_t decode_workspace_bytes(int layers, int b, int G);
int launch_decode_step(int layers, int b, int H, int N, int G, int act, int io, float* h,
                       float* conv_state, const void* xbc, const float* dt, const float* A,
                       const float* D, const float* conv_w, const float* conv_b, void* y,
                       void* ws, cudaStream_t s);
int create_decode_plan(ssd_decode_plan** out, int layers, int b, int H, int N, int G, int act,
                       int io, float* h, float* conv_state, const void* xbc_ring,
                       const float* dt_ring, int ring, const float* A, const float* D,
                       const float* conv_w, const float* conv_b, void* y_ring, int n_steps,
                       void* ws);
int launch_decode_plan(ssd_decode_plan* plan, cudaStream_t s);
int destroy_decode_plan(ssd_decode_plan* plan);
int decode_noalloc_scratch(void** ptr, size_t* bytes);

static thread_local char g_detail[512];

int set_error(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return status;
}

int cuda_status(cudaError_t e, const char* where) {
    return set_error(SSD_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

// The dynamic shared-memory limit is a per-device attribute of a kernel: set it once per
// (kernel, device, size) instead of on every launch (a host call each time).
int smem_limit_once(const void* func, int bytes) {
    static std::mutex mu;
    static std::vector<std::tuple<const void*, int, int>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(mu);
    for (const auto& d : done)
        if (std::get<0>(d) == func && std::get<1>(d) == dev && std::get<2>(d) >= bytes) return SSD_OK;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(MaxDynamicSharedMemorySize)");
    // the single-GPU prefill kernels all ask for the largest shared-memory carveout, so that
    // the small ones launched between large ones leave the SMs' L1/shared split as it is
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute(PreferredSharedMemoryCarveout)");
    done.emplace_back(func, dev, bytes);
    return SSD_OK;
}

// ---- launch accounting and event timing
namespace {
constexpr int kMaxProf = 65536;
std::atomic<uint64_t> g_launches{0};
bool g_prof = false;
int g_prof_n = 0;
int g_open = -1;
std::vector<cudaEvent_t> g_ev;     // 2 per recorded launch, created on demand and reused
std::vector<int> g_rec_name;       // name index per recorded launch
std::vector<std::string> g_names;  // distinct names in first-launch order
}  // namespace

void count_launches(uint64_t n) { g_launches += n; }

void prof_start(const char* name, cudaStream_t s) {
    if (!g_prof || g_prof_n >= kMaxProf) return;
    int idx = -1;
    for (size_t i = 0; i < g_names.size(); ++i)
        if (g_names[i] == name) { idx = (int)i; break; }
    if (idx < 0) { g_names.emplace_back(name); idx = (int)g_names.size() - 1; }
    while ((int)g_ev.size() < 2 * (g_prof_n + 1)) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return;
        g_ev.push_back(e);
    }
    if ((int)g_rec_name.size() <= g_prof_n) g_rec_name.resize(g_prof_n + 1);
    g_rec_name[g_prof_n] = idx;
    cudaEventRecord(g_ev[2 * g_prof_n], s);
    g_open = g_prof_n;
}

void prof_stop(cudaStream_t s) {
    if (!g_prof || g_open < 0) return;
    cudaEventRecord(g_ev[2 * g_open + 1], s);
    g_prof_n = g_open + 1;
    g_open = -1;
}

namespace {

constexpr int kMaxGridYZ = 65535;

struct Range {
    const void* p;
    size_t n;
};

bool overlaps(Range a, Range b) {
    if (!a.p || !b.p || a.n == 0 || b.n == 0) return false;
    const uintptr_t a0 = (uintptr_t)a.p, b0 = (uintptr_t)b.p;
    return a0 < b0 + b.n && b0 < a0 + a.n;
}

int check_ptr(const void* p, const char* name, bool required) {
    if (!p) {
        if (required) return set_error(SSD_ERR_INVALID_ARG, "%s is NULL", name);
        return SSD_OK;
    }
    if (!aligned16(p)) return set_error(SSD_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return SSD_OK;
}

#define SSD_CHECK(expr)                 \
    do {                                \
        int st_ = (expr);               \
        if (st_ != SSD_OK) return st_;  \
    } while (0)

int check_prefill_shape(int b, int T, int H, int P, int N, int G, int chunk, int io) {
    if (io != SSD_F32 && io != SSD_BF16) return set_error(SSD_ERR_INVALID_ARG, "io_dtype %d is not SSD_F32/SSD_BF16", io);
    if (b < 0 || T < 0) return set_error(SSD_ERR_INVALID_ARG, "negative size b=%d T=%d", b, T);
    if (H < 1 || P < 1 || N < 1 || G < 1) return set_error(SSD_ERR_INVALID_ARG, "H, P, N, G must be >= 1 (H=%d P=%d N=%d G=%d)", H, P, N, G);
    if (H % G) return set_error(SSD_ERR_INVALID_ARG, "H=%d is not a multiple of G=%d", H, G);
    if (chunk != 64 && chunk != 128 && chunk != 256) return set_error(SSD_ERR_INVALID_ARG, "chunk=%d not in {64,128,256}", chunk);
    if (P != 64) return set_error(SSD_ERR_UNSUPPORTED, "P=%d (only 64 is implemented)", P);
    if (N != 64 && N != 128) return set_error(SSD_ERR_UNSUPPORTED, "N=%d (only 64 and 128 are implemented)", N);
    if (H > kMaxGridYZ || b > kMaxGridYZ) return set_error(SSD_ERR_UNSUPPORTED, "H=%d or b=%d above 65535", H, b);
    return SSD_OK;
}

}  // namespace
}  // namespace ssd

using namespace ssd;

extern "C" {

int ssd_version(void) { return 100; }

const char* ssd_status_string(int status) {
    switch (status) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape not implemented";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA call failed";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: bounded device wait expired";
        case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
        case SSD_ERR_INTERNAL: return "SSD_ERR_INTERNAL: device consistency check failed";
        default: return "unknown ssd_status";
    }
}

const char* ssd_last_error(void) { return g_detail; }

uint64_t ssd_launch_count(void) { return g_launches.load(); }

int ssd_profile_begin(void) {
    g_prof = true;
    g_prof_n = 0;
    g_open = -1;
    g_names.clear();
    return SSD_OK;
}

int ssd_profile_end(ssd_kernel_time* out, int max_entries) {
    g_prof = false;
    std::vector<double> tot(g_names.size(), 0.0);
    std::vector<int> cnt(g_names.size(), 0);
    for (int i = 0; i < g_prof_n; ++i) {
        cudaError_t e = cudaEventSynchronize(g_ev[2 * i + 1]);
        float ms = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, g_ev[2 * i], g_ev[2 * i + 1]);
        if (e != cudaSuccess) return -cuda_status(e, "ssd_profile_end");
        tot[g_rec_name[i]] += ms;
        cnt[g_rec_name[i]] += 1;
    }
    int n = 0;
    for (size_t k = 0; k < g_names.size() && n < max_entries && out; ++k, ++n) {
        snprintf(out[n].name, sizeof(out[n].name), "%s", g_names[k].c_str());
        out[n].launches = cnt[k];
        out[n].total_ms = tot[k];
    }
    g_prof_n = 0;
    return n;
}

// Prefill workspace: [0, 256) device status word, then the path's scratch.
static constexpr size_t kStatusBytes = 256;

// ssd_debug_force_fma_prefill: every prefill takes the fp32-FMA path
static std::atomic<int> g_force_fma{0};
static bool use_tc(int P, int N, int io) { return prefill_tc_supported(P, N, io) && !g_force_fma.load(); }

static size_t prefill_ws_bytes(int b, int T, int H, int P, int N, int chunk, int io) {
    if (use_tc(P, N, io)) return kStatusBytes + prefill_tc_workspace_bytes(b, T, H);
    return kStatusBytes + prefill_simt_workspace_bytes(b, T, H, N, chunk, io);
}

size_t ssd_prefill_workspace_size(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype) {
    if (check_prefill_shape(b, T, H, P, N, G, chunk, io_dtype) != SSD_OK) return 0;
    if (b == 0 || T == 0) return 0;
    return prefill_ws_bytes(b, T, H, P, N, chunk, io_dtype);
}

int ssd_debug_starve_next_prefill(unsigned long long wait_limit_ns) {
    g_detail[0] = 0;
    if (wait_limit_ns < 1000000ull || wait_limit_ns > 10000000000ull)
        return set_error(SSD_ERR_INVALID_ARG, "wait_limit_ns %llu outside [1e6, 1e10]", wait_limit_ns);
    prefill_tc_starve_next(wait_limit_ns);
    return SSD_OK;
}

int ssd_prefill_segments(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype) {
    if (check_prefill_shape(b, T, H, P, N, G, chunk, io_dtype) != SSD_OK) return 0;
    if (b == 0 || T == 0 || !use_tc(P, N, io_dtype)) return 1;
    return prefill_tc_segments(b, T, H);
}

int ssd_prefill_whole_units(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype) {
    if (check_prefill_shape(b, T, H, P, N, G, chunk, io_dtype) != SSD_OK) return -1;
    if (b == 0 || T == 0 || !use_tc(P, N, io_dtype)) return b * H;
    return prefill_tc_whole_units(b, T, H);
}

size_t ssd_prefill_local_state_workspace_size(int b, int T, int H, int P, int N, int G, int io_dtype) {
    if (check_prefill_shape(b, T, H, P, N, G, 256, io_dtype) != SSD_OK || !prefill_tc_supported(P, N, io_dtype))
        return 0;
    if (b == 0 || T == 0) return 0;
    return prefill_tc_local_state_workspace_bytes(b, T, H);
}

int ssd_prefill_local_state(int b, int T, int H, int P, int N, int G, int io_dtype, const void* x, const float* dt,
                            const float* A, const void* B, float* h_local, float* log_decay, void* workspace,
                            size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    SSD_CHECK(check_prefill_shape(b, T, H, P, N, G, 256, io_dtype));
    if (!prefill_tc_supported(P, N, io_dtype))
        return set_error(SSD_ERR_UNSUPPORTED, "local state: tensor-core shapes only (bf16, P = 64, N = 128)");
    SSD_CHECK(check_ptr(h_local, "h_local", true));
    SSD_CHECK(check_ptr(log_decay, "log_decay", true));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)b * H * P * N * sizeof(float), ld_bytes = (size_t)b * H * sizeof(float);
    if (overlaps({h_local, state_bytes}, {log_decay, ld_bytes}))
        return set_error(SSD_ERR_INVALID_ARG, "h_local overlaps log_decay");
    if (b == 0) return SSD_OK;
    if (T == 0) {  // no tokens: nothing accumulates and nothing decays
        SSD_CUDA_TRY(cudaMemsetAsync(h_local, 0, state_bytes, s));
        SSD_CUDA_TRY(cudaMemsetAsync(log_decay, 0, ld_bytes, s));
        return SSD_OK;
    }
    SSD_CHECK(check_ptr(x, "x", true));
    SSD_CHECK(check_ptr(dt, "dt", true));
    SSD_CHECK(check_ptr(A, "A", true));
    SSD_CHECK(check_ptr(B, "B", true));
    const Range outs[] = {{h_local, state_bytes}, {log_decay, ld_bytes}};
    const Range rin[] = {{x, (size_t)b * T * H * P * 2}, {B, (size_t)b * T * G * N * 2}, {dt, (size_t)b * T * H * 4},
                         {A, (size_t)H * 4}};
    for (const Range& o : outs)
        for (const Range& i : rin)
            if (overlaps(o, i)) return set_error(SSD_ERR_INVALID_ARG, "an output overlaps an input");
    const size_t need = prefill_tc_local_state_workspace_bytes(b, T, H);
    if (!workspace || workspace_bytes < need)
        return set_error(SSD_ERR_WORKSPACE, "workspace %zu bytes at %p, need %zu", workspace_bytes, workspace, need);
    if (!aligned16(workspace)) return set_error(SSD_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    for (const Range& o : outs)
        if (overlaps({workspace, need}, o)) return set_error(SSD_ERR_INVALID_ARG, "workspace overlaps an output");
    for (const Range& i : rin)
        if (overlaps({workspace, need}, i)) return set_error(SSD_ERR_INVALID_ARG, "workspace overlaps an input");
    return launch_prefill_tc_local_state(b, T, H, G, x, dt, A, B, h_local, log_decay, workspace, s);
}

int ssd_prefill_context_scan(int world, int rank, int b, int H, int P, int N, const float* h0, const float* h_local_all,
                             const float* log_decay_all, float* h_in, void* stream) {
    g_detail[0] = 0;
    if (world < 1 || rank < 0 || rank >= world)
        return set_error(SSD_ERR_INVALID_ARG, "rank %d outside [0, world=%d)", rank, world);
    if (b < 0 || H < 1) return set_error(SSD_ERR_INVALID_ARG, "b=%d H=%d", b, H);
    if (P != 64 || N != 128) return set_error(SSD_ERR_UNSUPPORTED, "context scan: P = 64, N = 128 only");
    if (H > kMaxGridYZ || b > kMaxGridYZ) return set_error(SSD_ERR_UNSUPPORTED, "H=%d or b=%d above 65535", H, b);
    SSD_CHECK(check_ptr(h0, "h0", false));
    SSD_CHECK(check_ptr(h_in, "h_in", true));
    if (rank > 0) {
        SSD_CHECK(check_ptr(h_local_all, "h_local_all", true));
        SSD_CHECK(check_ptr(log_decay_all, "log_decay_all", true));
    }
    const size_t state_bytes = (size_t)b * H * P * N * sizeof(float);
    if (overlaps({h_in, state_bytes}, {h_local_all, (size_t)world * state_bytes}) ||
        overlaps({h_in, state_bytes}, {log_decay_all, (size_t)world * b * H * 4}) ||
        (h0 && h0 != h_in && overlaps({h_in, state_bytes}, {h0, state_bytes})))
        return set_error(SSD_ERR_INVALID_ARG, "h_in overlaps an input (only exact aliasing of h0 is allowed)");
    if (b == 0) return SSD_OK;
    return launch_context_scan(rank, b, H, h0, h_local_all, log_decay_all, h_in, static_cast<cudaStream_t>(stream));
}

int ssd_debug_decay_precision(int mode) {
    g_detail[0] = 0;
    if (mode < 0 || mode > 2) return set_error(SSD_ERR_INVALID_ARG, "decay precision mode %d is not 0, 1 or 2", mode);
    prefill_tc_decay_mode(mode);
    return SSD_OK;
}

int ssd_debug_force_prefill_split(int n_full, int nseg) {
    g_detail[0] = 0;
    if (n_full < 0 || nseg < 0) return set_error(SSD_ERR_INVALID_ARG, "n_full %d / nseg %d negative", n_full, nseg);
    prefill_tc_force_split(n_full, nseg);
    return SSD_OK;
}

int ssd_debug_force_fma_prefill(int on) {
    g_detail[0] = 0;
    if (on != 0 && on != 1) return set_error(SSD_ERR_INVALID_ARG, "on is %d, not 0 or 1", on);
    g_force_fma.store(on);
    return SSD_OK;
}

int ssd_debug_force_prefill_segments(int nseg) {
    g_detail[0] = 0;
    if (nseg < 0) return set_error(SSD_ERR_INVALID_ARG, "nseg %d is negative", nseg);
    prefill_tc_force_segments(nseg);
    return SSD_OK;
}

int ssd_prefill_check(void* workspace, void* stream) {
    g_detail[0] = 0;
    if (!workspace) return set_error(SSD_ERR_INVALID_ARG, "workspace is NULL");
    return prefill_tc_status(workspace, static_cast<cudaStream_t>(stream));
}

static int prefill_impl(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype, const void* x,
                        const float* dt, const DtMap& dtm, const float* A, const void* B, const void* C,
                        const float* D, const float* h0, void* y, float* h_final, void* workspace,
                        size_t workspace_bytes, void* stream) {
    SSD_CHECK(check_prefill_shape(b, T, H, P, N, G, chunk, io_dtype));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)b * H * P * N * sizeof(float);
    SSD_CHECK(check_ptr(h0, "h0", false));
    SSD_CHECK(check_ptr(h_final, "h_final", false));
    if (h0 && h_final && h0 != h_final && overlaps({h0, state_bytes}, {h_final, state_bytes}))
        return set_error(SSD_ERR_INVALID_ARG, "h_final partially overlaps h0 (only exact aliasing is allowed)");
    if (b == 0) return SSD_OK;
    if (T == 0) {  // no tokens: the state passes through unchanged
        if (h_final && h_final != h0) {
            if (h0) SSD_CUDA_TRY(cudaMemcpyAsync(h_final, h0, state_bytes, cudaMemcpyDeviceToDevice, s));
            else SSD_CUDA_TRY(cudaMemsetAsync(h_final, 0, state_bytes, s));
        }
        return SSD_OK;
    }
    SSD_CHECK(check_ptr(x, "x", true));
    SSD_CHECK(check_ptr(dt, "dt", true));
    SSD_CHECK(check_ptr(A, "A", true));
    SSD_CHECK(check_ptr(B, "B", true));
    SSD_CHECK(check_ptr(C, "C", true));
    SSD_CHECK(check_ptr(D, "D", true));
    SSD_CHECK(check_ptr(y, "y", true));
    const size_t io_b = io_dtype == SSD_BF16 ? 2 : 4;
    const Range ry{y, (size_t)b * T * H * P * io_b};
    const Range rin[] = {{x, (size_t)b * T * H * P * io_b}, {B, (size_t)b * T * G * N * io_b},
                         {C, (size_t)b * T * G * N * io_b}, {dt, (size_t)b * T * H * 4},
                         {A, (size_t)H * 4}, {D, (size_t)H * 4}, {h0, h0 ? state_bytes : 0}};
    const char* names[] = {"x", "B", "C", "dt", "A", "D", "h0"};
    for (int i = 0; i < 7; ++i) {
        if (overlaps(ry, rin[i])) return set_error(SSD_ERR_INVALID_ARG, "y overlaps input %s", names[i]);
        if (i < 6 && overlaps({h_final, h_final ? state_bytes : 0}, rin[i]))
            return set_error(SSD_ERR_INVALID_ARG, "h_final overlaps input %s", names[i]);
    }
    if (overlaps(ry, {h_final, h_final ? state_bytes : 0})) return set_error(SSD_ERR_INVALID_ARG, "y overlaps h_final");
    const size_t need = prefill_ws_bytes(b, T, H, P, N, chunk, io_dtype);
    if (!workspace || workspace_bytes < need)
        return set_error(SSD_ERR_WORKSPACE, "workspace %zu bytes at %p, need %zu", workspace_bytes, workspace, need);
    if (!aligned16(workspace)) return set_error(SSD_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    if (overlaps({workspace, need}, ry)) return set_error(SSD_ERR_INVALID_ARG, "workspace overlaps y");
    if (overlaps({workspace, need}, {h_final, h_final ? state_bytes : 0}))
        return set_error(SSD_ERR_INVALID_ARG, "workspace overlaps h_final");
    for (int i = 0; i < 7; ++i)
        if (overlaps({workspace, need}, rin[i])) return set_error(SSD_ERR_INVALID_ARG, "workspace overlaps %s", names[i]);
    if (use_tc(P, N, io_dtype))
        return launch_prefill_tc(b, T, H, G, x, dt, dtm, A, B, C, D, h0, y, h_final, workspace, s);
    SSD_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(int), s));
    return launch_prefill_simt(b, T, H, N, G, chunk, io_dtype, x, dt, dtm, A, B, C, D, h0, y, h_final,
                               static_cast<char*>(workspace) + kStatusBytes, s);
}

int ssd_prefill(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype,
                const void* x, const float* dt, const float* A, const void* B, const void* C,
                const float* D, const float* h0, void* y, float* h_final, void* workspace,
                size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    const DtMap plain{nullptr, 0.f, 0.f, 0};
    return prefill_impl(b, T, H, P, N, G, chunk, io_dtype, x, dt, plain, A, B, C, D, h0, y, h_final, workspace,
                        workspace_bytes, stream);
}

int ssd_prefill_dt_raw(int b, int T, int H, int P, int N, int G, int chunk, int io_dtype,
                       const void* x, const float* dt_raw, const float* dt_bias, float dt_min, float dt_max,
                       const float* A, const void* B, const void* C, const float* D, const float* h0,
                       void* y, float* h_final, void* workspace, size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    if (!(dt_min >= 0.f) || !(dt_max > dt_min))  // also rejects NaN limits
        return set_error(SSD_ERR_INVALID_ARG, "dt clamp range [%g, %g] must satisfy 0 <= dt_min < dt_max",
                         (double)dt_min, (double)dt_max);
    SSD_CHECK(check_ptr(dt_bias, "dt_bias", false));
    if (dt_bias && H > 0 && overlaps({dt_bias, (size_t)H * 4}, {y, (size_t)b * T * H * P * (io_dtype == SSD_BF16 ? 2 : 4)}))
        return set_error(SSD_ERR_INVALID_ARG, "y overlaps input dt_bias");
    const DtMap raw{dt_bias, dt_min, dt_max, 1};
    return prefill_impl(b, T, H, P, N, G, chunk, io_dtype, x, dt_raw, raw, A, B, C, D, h0, y, h_final, workspace,
                        workspace_bytes, stream);
}

size_t ssd_decode_workspace_size(int layers, int b, int G) {
    if (layers < 1 || b < 1 || G < 1) return 0;
    return decode_workspace_bytes(layers, b, G);
}

static int check_decode(int layers, int b, int H, int P, int N, int G, int kconv, int act, int io,
                        const float* h, const float* conv_state, const float* A, const float* D,
                        const float* conv_w, const float* conv_b, void* ws, size_t ws_bytes) {
    if (io != SSD_F32 && io != SSD_BF16) return set_error(SSD_ERR_INVALID_ARG, "io_dtype %d is not SSD_F32/SSD_BF16", io);
    if (act != SSD_ACT_NONE && act != SSD_ACT_SILU) return set_error(SSD_ERR_INVALID_ARG, "act %d is not SSD_ACT_NONE/SSD_ACT_SILU", act);
    if (layers < 0 || b < 0) return set_error(SSD_ERR_INVALID_ARG, "negative size layers=%d b=%d", layers, b);
    if (H < 1 || P < 1 || N < 1 || G < 1) return set_error(SSD_ERR_INVALID_ARG, "H, P, N, G must be >= 1");
    if (H % G) return set_error(SSD_ERR_INVALID_ARG, "H=%d is not a multiple of G=%d", H, G);
    if (kconv < 1) return set_error(SSD_ERR_INVALID_ARG, "kconv=%d must be >= 1", kconv);
    if (kconv != 4) return set_error(SSD_ERR_UNSUPPORTED, "kconv=%d (only 4 is implemented)", kconv);
    if (P != 64) return set_error(SSD_ERR_UNSUPPORTED, "P=%d (only 64 is implemented)", P);
    if (N != 64 && N != 128) return set_error(SSD_ERR_UNSUPPORTED, "N=%d (only 64 and 128 are implemented)", N);
    if (layers > kMaxGridYZ || b > kMaxGridYZ) return set_error(SSD_ERR_UNSUPPORTED, "layers or b above 65535");
    if (layers == 0 || b == 0) return SSD_OK;
    SSD_CHECK(check_ptr(h, "h", true));
    SSD_CHECK(check_ptr(conv_state, "conv_state", true));
    SSD_CHECK(check_ptr(A, "A", true));
    SSD_CHECK(check_ptr(D, "D", true));
    SSD_CHECK(check_ptr(conv_w, "conv_w", true));
    SSD_CHECK(check_ptr(conv_b, "conv_b", true));
    const size_t need = decode_workspace_bytes(layers, b, G);
    if (!ws || ws_bytes < need) return set_error(SSD_ERR_WORKSPACE, "workspace %zu bytes at %p, need %zu", ws_bytes, ws, need);
    if (!aligned16(ws)) return set_error(SSD_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    return SSD_OK;
}

// The buffers a decode step writes (h, conv_state, y and the workspace's arrival counters)
// must not overlap one another or any buffer the step reads (xbc, dt, A, D, conv_w, conv_b);
// for a plan, xbc, dt and y hold `ring` steps.
static int check_decode_overlaps(int layers, int b, int H, int P, int N, int G, int kconv, int io_dtype,
                                 const float* h, const float* conv_state, const void* xbc, const float* dt,
                                 const float* A, const float* D, const float* conv_w, const float* conv_b,
                                 const void* y, int ring, const void* ws) {
    const size_t io_b = io_dtype == SSD_BF16 ? 2 : 4;
    const size_t Dc = (size_t)H * P + 2 * (size_t)G * N, lb = (size_t)layers * b, R = (size_t)ring;
    const Range writes[] = {{h, lb * H * P * N * 4}, {conv_state, lb * Dc * (kconv - 1) * 4},
                            {y, R * lb * H * P * io_b}, {ws, decode_workspace_bytes(layers, b, G)}};
    const Range reads[] = {{xbc, R * lb * Dc * io_b},         {dt, R * lb * H * 4},
                           {A, (size_t)layers * H * 4},       {D, (size_t)layers * H * 4},
                           {conv_w, (size_t)layers * Dc * kconv * 4}, {conv_b, (size_t)layers * Dc * 4}};
    const char* wname[] = {"h", "conv_state", "y", "workspace"};
    const char* rname[] = {"xbc", "dt", "A", "D", "conv_w", "conv_b"};
    for (int i = 0; i < 4; ++i) {
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(writes[i], writes[j]))
                return set_error(SSD_ERR_INVALID_ARG, "%s overlaps %s", wname[i], wname[j]);
        for (int j = 0; j < 6; ++j)
            if (overlaps(writes[i], reads[j]))
                return set_error(SSD_ERR_INVALID_ARG, "%s overlaps %s", wname[i], rname[j]);
    }
    return SSD_OK;
}

int ssd_decode_step(int layers, int b, int H, int P, int N, int G, int kconv, int act, int io_dtype,
                    float* h, float* conv_state, const void* xbc, const float* dt, const float* A,
                    const float* D, const float* conv_w, const float* conv_b, void* y,
                    void* workspace, size_t workspace_bytes, void* stream) {
    g_detail[0] = 0;
    SSD_CHECK(check_decode(layers, b, H, P, N, G, kconv, act, io_dtype, h, conv_state, A, D, conv_w,
                           conv_b, workspace, workspace_bytes));
    if (layers == 0 || b == 0) return SSD_OK;
    SSD_CHECK(check_ptr(xbc, "xbc", true));
    SSD_CHECK(check_ptr(dt, "dt", true));
    SSD_CHECK(check_ptr(y, "y", true));
    SSD_CHECK(check_decode_overlaps(layers, b, H, P, N, G, kconv, io_dtype, h, conv_state, xbc, dt, A, D, conv_w,
                                    conv_b, y, 1, workspace));
    return launch_decode_step(layers, b, H, N, G, act, io_dtype, h, conv_state, xbc, dt, A, D, conv_w,
                              conv_b, y, workspace, static_cast<cudaStream_t>(stream));
}

int ssd_decode_step_noalloc(int layers, int b, int H, int P, int N, int G, int kconv, int act,
                            int io_dtype, float* h, float* conv_state, const void* xbc,
                            const float* dt, const float* A, const float* D, const float* conv_w,
                            const float* conv_b, void* y, void* stream) {
    g_detail[0] = 0;
    if (layers > 0 && b > 0 && G > 0 &&
        (size_t)layers * (size_t)b * (size_t)G > (size_t)SSD_DECODE_NOALLOC_MAX_COUNTERS)
        return set_error(SSD_ERR_INVALID_ARG,
                         "layers*b*G = %zu exceeds the %d arrival counters of the allocation-free decode step",
                         (size_t)layers * b * G, SSD_DECODE_NOALLOC_MAX_COUNTERS);
    void* scratch = nullptr;
    size_t cap = 0;
    if (layers > 0 && b > 0) SSD_CHECK(decode_noalloc_scratch(&scratch, &cap));
    // the library's own scratch stands in for the caller workspace of ssd_decode_step
    return ssd_decode_step(layers, b, H, P, N, G, kconv, act, io_dtype, h, conv_state, xbc, dt, A, D,
                           conv_w, conv_b, y, scratch, cap, stream);
}

int ssd_decode_plan_create(ssd_decode_plan** plan, int layers, int b, int H, int P, int N, int G,
                           int kconv, int act, int io_dtype, float* h, float* conv_state,
                           const void* xbc_ring, const float* dt_ring, int ring, const float* A,
                           const float* D, const float* conv_w, const float* conv_b, void* y_ring,
                           int n_steps, void* workspace, size_t workspace_bytes) {
    g_detail[0] = 0;
    if (!plan) return set_error(SSD_ERR_INVALID_ARG, "plan is NULL");
    *plan = nullptr;
    SSD_CHECK(check_decode(layers, b, H, P, N, G, kconv, act, io_dtype, h, conv_state, A, D, conv_w,
                           conv_b, workspace, workspace_bytes));
    if (layers == 0 || b == 0) return set_error(SSD_ERR_INVALID_ARG, "a decode plan needs layers >= 1 and b >= 1");
    if (ring < 1) return set_error(SSD_ERR_INVALID_ARG, "ring=%d must be >= 1", ring);
    if (n_steps < 0) return set_error(SSD_ERR_INVALID_ARG, "n_steps=%d must be >= 0", n_steps);
    SSD_CHECK(check_ptr(xbc_ring, "xbc_ring", true));
    SSD_CHECK(check_ptr(dt_ring, "dt_ring", true));
    SSD_CHECK(check_ptr(y_ring, "y_ring", true));
    SSD_CHECK(check_decode_overlaps(layers, b, H, P, N, G, kconv, io_dtype, h, conv_state, xbc_ring, dt_ring, A, D,
                                    conv_w, conv_b, y_ring, ring, workspace));
    return create_decode_plan(plan, layers, b, H, N, G, act, io_dtype, h, conv_state, xbc_ring, dt_ring,
                              ring, A, D, conv_w, conv_b, y_ring, n_steps, workspace);
}

int ssd_decode_plan_launch(ssd_decode_plan* plan, void* stream) {
    g_detail[0] = 0;
    if (!plan) return set_error(SSD_ERR_INVALID_ARG, "plan is NULL");
    return launch_decode_plan(plan, static_cast<cudaStream_t>(stream));
}

int ssd_decode_plan_destroy(ssd_decode_plan* plan) {
    g_detail[0] = 0;
    if (!plan) return SSD_OK;
    return destroy_decode_plan(plan);
}

int ssd_decode_loop(int layers, int b, int H, int P, int N, int G, int kconv, int act, int io_dtype, float* h,
                    float* conv_state, const void* xbc_ring, const float* dt_ring, int ring, const float* A,
                    const float* D, const float* conv_w, const float* conv_b, void* y_ring, int n_steps,
                    void* workspace, size_t workspace_bytes, void* stream) {
    ssd_decode_plan* plan = nullptr;
    SSD_CHECK(ssd_decode_plan_create(&plan, layers, b, H, P, N, G, kconv, act, io_dtype, h, conv_state, xbc_ring,
                                     dt_ring, ring, A, D, conv_w, conv_b, y_ring, n_steps, workspace,
                                     workspace_bytes));
    const int st = ssd_decode_plan_launch(plan, stream);
    // an executable graph destroyed while in flight is freed when it completes
    const int st2 = destroy_decode_plan(plan);
    return st != SSD_OK ? st : st2;
}

}  // extern "C"
