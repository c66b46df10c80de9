// gemm.h -- internal interface of the tcgen05 GEMM (k_gemm.cu) and its
// fused epilogues.
#pragma once

#include "common.cuh"

namespace ret {

enum : int {
    kEpiStore = 0,            // out = scale * acc
    kEpiRotate = 1,           // out = rot(scale * acc)             (queries)
    kEpiRotateScaleZeta = 2,  // out = rot(scale * acc) * zeta      (keys)
    kEpiSwish = 3,            // out = swish(acc)                   (gate)
    kEpiGelu = 4,             // out = gelu(acc)                    (FFN hidden layer)
    kEpiResidual = 5,         // out = scale * acc + res            (a residual branch)
};

struct GemmSegment {
    const void* B;  // [K, N] bf16 row-major
    int N;
};

struct GemmSegOut {
    void* ptr;          // [M, ld] row-major destination of this segment
    int ld;             // leading dimension (elements)
    int kind;           // kEpi*
    ret_dtype dtype;    // RET_F32 or RET_BF16 (rotations: bf16); ld * element size a multiple of 16 bytes
    float scale;
    int head_dim;       // rotations: width of a head (pairs rotate within it)
    const __nv_bfloat16* res;  // kEpiResidual: [M, res_ld] bf16 added to the result
    int res_ld;
};

struct GemmEpilogue {
    GemmSegOut seg[4];
    int M;                  // filled by launch_gemm
    int seq;                // rows are (batch, token) with token = row % seq
    int chunk;              // chunk length for the zeta of the keys
    int xpos;               // rotations: 0 leaves the pairs unrotated
    long long pos_offset;
    double log2base;        // log2(theta_base)
    // Rotations: (cos, sin) of every (token, pair) at position pos_offset +
    // token, [seq][head_dim / 2] fp32, 16-byte aligned; required when xpos
    // rotates a segment (head_dim a multiple of 32).
    const float2* rot_cs;
    double log2g[kMaxHeads];
};

// C = A B with A [M, K] bf16 row-major and B split into column segments.
ret_status launch_gemm(const void* A, int M, int K, const GemmSegment* segs, int nseg, const GemmEpilogue& epi,
                       cudaStream_t s);

cudaError_t read_clear_error_gemm(int* flag);

}  // namespace ret
