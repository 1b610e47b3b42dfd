// common.cuh -- small shared helpers for the sm_100a SSD kernels (no method arithmetic
// beyond type conversion lives here).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/ssd.h"

namespace ssd {

// Records a detail string for ssd_last_error() and returns the status unchanged.
int set_error(int status, const char* fmt, ...);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Load one io element as float.
__device__ __forceinline__ float load_io(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_io(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_io(float* p, size_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_io(__nv_bfloat16* p, size_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
}

// Time step as the prefill kernels read it.  By default dt arrives already positive (the
// softplus applied by the caller) and is used as is.  With `raw` set, the kernels apply the
// pre-processing of the Mamba-2 block where they load it, so the raw projection output
// never takes a separate pass over memory ("Compiler-First State Space Duality and
// Portable O(1) Autoregressive Caching": the elementwise chain ahead of the SSD fused into
// the kernel): dt = clamp(softplus(dt_raw + bias[h]), lo, hi), softplus(z) = log(1 + e^z)
// (taken as z above 20, where the two differ by less than fp32 rounding).
struct DtMap {
    const float* bias;  // [H] or nullptr (zero bias)
    float lo, hi;       // clamp range (hi may be +inf)
    int raw;            // 0: dt is used as given
};
// clamp(softplus(z)) for z = dt_raw + the head's bias
__device__ __forceinline__ float dt_softplus_clamp(float z, const DtMap& m) {
    const float sp = z > 20.f ? z : log1pf(expf(z));
    return fminf(fmaxf(sp, m.lo), m.hi);
}
__device__ __forceinline__ float dt_value(float v, const DtMap& m, int h) {
    if (!m.raw) return v;
    return dt_softplus_clamp(v + (m.bias ? __ldg(m.bias + h) : 0.f), m);
}

// Map a CUDA error to a status with detail.
int cuda_status(cudaError_t e, const char* where);

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current device, once.
int smem_limit_once(const void* func, int bytes);

// Launch accounting and optional per-kernel event timing (see ssd_profile_begin).
void count_launches(uint64_t n);
void prof_start(const char* name, cudaStream_t s);  // no-op unless profiling
void prof_stop(cudaStream_t s);

// Brackets one launch: counts it and, when profiling, records events around it.
struct LaunchScope {
    cudaStream_t s;
    LaunchScope(const char* name, cudaStream_t st, uint64_t n = 1) : s(st) {
        count_launches(n);
        prof_start(name, st);
    }
    ~LaunchScope() { prof_stop(s); }
};

}  // namespace ssd

#define SSD_CUDA_TRY(expr)                                                   \
    do {                                                                     \
        cudaError_t e_ = (expr);                                             \
        if (e_ != cudaSuccess) return ::ssd::cuda_status(e_, #expr);         \
    } while (0)
