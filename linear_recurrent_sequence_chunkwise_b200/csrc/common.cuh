// common.cuh -- small device and host helpers shared by the library's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "retention.h"

namespace ret {

// ---------------------------------------------------------------- host side

// Record a failure message for the calling thread and return `st`.
ret_status fail(ret_status st, const char* fmt, ...);
// Map the last launch error (if any) to RET_ERR_CUDA.
ret_status check_launch(const char* what);

// Per-head constants, computed on the host in fp64 and passed by value.
constexpr int kMaxHeads = 128;
struct HeadConsts {
    double log2g[kMaxHeads];  // log2(gamma_h); -inf for gamma_h = 0
    // Row a of a 128-row chunk the tensor-core kernels scale the decay about
    // (keys by gamma^(a-c), output rows by gamma^(r-a)): 127 when
    // gamma^128 >= 2^-60, 63 when gamma^64 >= 2^-100 (every factor then stays
    // within 2^+-100), -1 for a head the tensor-core kernels do not take.
    int anchor[kMaxHeads];
};
constexpr int kChunkAnchorFull = 127, kChunkAnchorMid = 63;
// The anchor rule above, for one head.
inline int decay_anchor(double log2g) {
    if (log2g * 128.0 >= -60.0) return kChunkAnchorFull;
    if (log2g * 64.0 >= -100.0) return kChunkAnchorMid;
    return -1;
}
// Fill `hc` from the host array; returns false if H is out of range.
bool make_head_consts(const double* gammas, int H, HeadConsts* hc);

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device-side error words: each translation unit whose kernels wait on
// mbarriers keeps its own word (no relocatable device code) and exposes a
// host reader that returns and clears it (cudaSuccess or the CUDA error).
constexpr int kErrTimeout = 1;
cudaError_t read_clear_error_chunk_ws(int* flag);

// ---------------------------------------------------------------- device side

__device__ __forceinline__ float ld_as_float(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_as_float(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

__device__ __forceinline__ void st_from_float(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_from_float(__nv_bfloat16* p, size_t i, float x) { p[i] = __float2bfloat16_rn(x); }

// gamma^e for integer e >= 0 with gamma^0 = 1 for every gamma (0^0 = 1):
// exp2 of e * log2(gamma) evaluated in fp64, rounded once to fp32.
__device__ __forceinline__ float gamma_pow_d(double log2g, long long e) {
    if (e == 0) return 1.0f;
    return (float)exp2((double)e * log2g);
}

// The rotation angle of pair p at position pos, reduced to [-pi, pi] in fp64
// and then rounded to fp32, so fp32 sincos sees a small argument.
__device__ __forceinline__ float rot_angle(long long pos, double theta) {
    const double two_pi = 6.283185307179586476925286766559;
    double a = (double)pos * theta;
    a -= two_pi * rint(a / two_pi);
    return (float)a;
}

}  // namespace ret
