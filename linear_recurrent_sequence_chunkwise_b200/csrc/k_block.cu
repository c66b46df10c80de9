// k_block.cu -- one RetNet block ("Hybrid Architectures: RetNet and the Three
// Computation Paradigms", section 9.2; RetNet paper summary, "Overall RetNet
// Architecture"): pre-LayerNorm residual layout
//     Y   = MSR(LN(X)) + X
//     out = FFN(LN(Y)) + Y,   FFN(x) = gelu(x W1) W2,  W1 [d, d_ff], W2 [d_ff, d]
// The MSR is the layer of k_msr.cu with the residual added in its output
// projection's epilogue; the FFN is two tcgen05 GEMMs with gelu and the
// residual fused into their epilogues; LayerNorm is one warp per row.
// Activations between the steps (LN outputs, Y, the FFN hidden layer) are
// bf16, every accumulation fp32.
#include <algorithm>
#include <cstring>

#include "gemm.h"
#include "kernels.h"

namespace ret {

namespace {

// One warp per row of x [M, d] (d a multiple of 8): mean, then the variance
// about it (biased), both in fp32 over the row held in L1; y = (x - mean) /
// sqrt(var + eps) * gain + bias in bf16.
__global__ void __launch_bounds__(256) k_layernorm(const __nv_bfloat16* __restrict__ x,
                                                   const __nv_bfloat16* __restrict__ gain,
                                                   const __nv_bfloat16* __restrict__ bias, __nv_bfloat16* __restrict__ y,
                                                   int M, int d, float eps) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= M) return;
    const __nv_bfloat16* xr = x + row * d;
    auto load8 = [&](int g, float* f) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr + 8 * g));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    };
    const int groups = d / 8;
    float s = 0.f;
    for (int g = lane; g < groups; g += 32) {
        float f[8];
        load8(g, f);
#pragma unroll
        for (int i = 0; i < 8; i++) s += f[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / d;
    float v = 0.f;
    for (int g = lane; g < groups; g += 32) {
        float f[8];
        load8(g, f);
#pragma unroll
        for (int i = 0; i < 8; i++) v = fmaf(f[i] - mean, f[i] - mean, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const float rstd = rsqrtf(v / d + eps);
    for (int g = lane; g < groups; g += 32) {
        float f[8];
        load8(g, f);
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            float a = (f[2 * i] - mean) * rstd, b = (f[2 * i + 1] - mean) * rstd;
            const int c = 8 * g + 2 * i;
            if (gain) {
                a *= __bfloat162float(gain[c]);
                b *= __bfloat162float(gain[c + 1]);
            }
            if (bias) {
                a += __bfloat162float(bias[c]);
                b += __bfloat162float(bias[c + 1]);
            }
            h[i] = __floats2bfloat162_rn(a, b);
        }
        *reinterpret_cast<uint4*>(y + row * d + 8 * g) = u;
    }
}

}  // namespace

ret_status launch_layernorm(const void* x, const void* gain, const void* bias, void* y, int M, int d, double eps,
                            cudaStream_t s) {
    const int blocks = (M + 7) / 8;
    k_layernorm<<<blocks, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(x),
                                       reinterpret_cast<const __nv_bfloat16*>(gain),
                                       reinterpret_cast<const __nv_bfloat16*>(bias),
                                       reinterpret_cast<__nv_bfloat16*>(y), M, d, (float)eps);
    return check_launch("layernorm");
}

size_t block_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv, int dff) {
    const size_t M = (size_t)B * N;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    // LN output (reused for LN2), Y, then the larger of the MSR scratch and the FFN hidden layer
    const size_t inner = std::max(msr_workspace_bytes(B, N, dmodel, H, dk, dv), M * (size_t)dff * 2);
    return al(M * dmodel * 2) + al(M * dmodel * 2) + al(inner);
}

ret_status launch_block(const BlockArgs& a, cudaStream_t s) {
    const MsrArgs& m0 = a.msr;
    const int M = m0.B * m0.N, d = m0.dmodel;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    uint8_t* w = reinterpret_cast<uint8_t*>(a.workspace);
    __nv_bfloat16* xn = reinterpret_cast<__nv_bfloat16*>(w);
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(w + al((size_t)M * d * 2));
    uint8_t* inner = w + 2 * al((size_t)M * d * 2);

    // 1. xn = LN1(X)
    ret_status st = launch_layernorm(m0.X, a.ln1_g, a.ln1_b, xn, M, d, a.ln_eps, s);
    if (st != RET_OK) return st;
    // 2. Y = MSR(xn) + X
    MsrArgs m = m0;
    m.X = xn;
    m.out = y;
    m.out_dt = RET_BF16;
    m.residual = m0.X;
    m.workspace = inner;
    if ((st = launch_msr(m, s)) != RET_OK) return st;
    // 3. xn = LN2(Y)
    if ((st = launch_layernorm(y, a.ln2_g, a.ln2_b, xn, M, d, a.ln_eps, s)) != RET_OK) return st;
    // 4. hidden = gelu(xn W1)
    __nv_bfloat16* hid = reinterpret_cast<__nv_bfloat16*>(inner);
    GemmSegment s1[1] = {{a.W1, a.dff}};
    GemmEpilogue e1;
    memset(&e1, 0, sizeof(e1));
    e1.seg[0] = {hid, a.dff, kEpiGelu, RET_BF16, 1.f, 0, nullptr, 0};
    e1.seq = m0.N;
    e1.chunk = 1;
    if ((st = launch_gemm(xn, M, d, s1, 1, e1, s)) != RET_OK) return st;
    // 5. out = hidden W2 + Y
    GemmSegment s2[1] = {{a.W2, d}};
    GemmEpilogue e2;
    memset(&e2, 0, sizeof(e2));
    e2.seg[0] = {a.out, d, kEpiResidual, a.out_dt, 1.f, 0, y, d};
    e2.seq = m0.N;
    e2.chunk = 1;
    return launch_gemm(hid, M, a.dff, s2, 1, e2, s);
}

}  // namespace ret
