// k_msr.cu -- the MultiScaleRetention layer ("Hybrid Architectures: RetNet
// and the Three Computation Paradigms", section 9.1; RetNet paper summary,
// "Gated Multi-Scale Retention"):
//     Q = rot(X W_Q), K = rot(k_scale X W_K), V = X W_V, G = X W_G
//     Y = Retention(Q, K, V)  per head with decay gamma_h
//     Z = swish(G) (.) GroupNorm_h(Y),   out = Z W_O
// as launches on one stream:
//   0. (xPos) the (cos, sin) of every (token, pair), once per call;
//   1. tcgen05 GEMM X [W_Q | W_K | W_V | W_G] whose epilogue writes the
//      rotated queries, the rotated keys already scaled by k_scale and by the
//      zeta decay of their place in the chunk (the chunkwise kernel's k'),
//      V, and swish(G), each bf16;
//   2. the chunkwise retention kernel on them, output fp32;
//   3. per-(token, head) GroupNorm over d_v (biased variance, eps inside the
//      square root, no affine) times swish(G), bf16, written over swish(G);
//   4. tcgen05 GEMM Z W_O.
#include "gemm.h"
#include "kernels.h"

namespace ret {

namespace {

// (cos, sin) of angle (pos0 + n) theta_p, theta_p = base^(-2p/head_dim), for
// n < seq, p < head_dim / 2; fp64 angle reduced to [-pi, pi], fp32 sincos.
__global__ void k_rot_table(float2* __restrict__ cs, int seq, int pairs, long long pos0, double log2base) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)seq * pairs) return;
    const int n = (int)(i / pairs), p = (int)(i % pairs);
    float s, c;
    sincosf(rot_angle(pos0 + n, exp2(-2.0 * p / (2 * pairs) * log2base)), &s, &c);
    cs[i] = make_float2(c, s);
}

// One warp per (token, head): d_v values, lanes own d_v / 32 consecutive
// elements each (d_v a multiple of 128, at most 1024).
template <int PER>
__global__ void __launch_bounds__(256) k_gn_gate(const float* __restrict__ Y, __nv_bfloat16* __restrict__ G, int rows,
                                                 int dv, float eps) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // (token, head)
    if (row >= rows) return;
    const float* y = Y + (size_t)row * dv + lane * PER;
    __nv_bfloat16* g = G + (size_t)row * dv + lane * PER;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; i += 4) {
        const float4 t = *reinterpret_cast<const float4*>(y + i);
        v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < PER; i++) s += v[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mu = s / dv;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const float d = v[i] - mu;
        q += d * d;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = rsqrtf(q / dv + eps);
#pragma unroll
    for (int i = 0; i < PER; i += 4) {  // 4 bf16 = 8 bytes, aligned since PER is a multiple of 4
        uint2 gw = *reinterpret_cast<const uint2*>(g + i);
        __nv_bfloat16* gb = reinterpret_cast<__nv_bfloat16*>(&gw);
        uint2 zw;
        __nv_bfloat16* zb = reinterpret_cast<__nv_bfloat16*>(&zw);
#pragma unroll
        for (int e = 0; e < 4; e++) zb[e] = __float2bfloat16_rn(__bfloat162float(gb[e]) * (v[i + e] - mu) * rstd);
        *reinterpret_cast<uint2*>(g + i) = zw;
    }
}

}  // namespace

size_t msr_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv) {
    (void)dmodel;
    const size_t M = (size_t)B * N;
    // q_rot, k' (bf16), v (bf16), swish(G) then Z (bf16), retention output
    // (fp32), the rotation's (cos, sin) table [N][dk/2]
    return M * H * ((size_t)dk * 2 * 2 + (size_t)dv * 2 * 2 + (size_t)dv * 4) + (size_t)N * (dk / 2) * 8 + 6 * 256;
}

ret_status launch_msr(const MsrArgs& m, cudaStream_t s) {
    const size_t M = (size_t)m.B * m.N;
    const int HK = m.H * m.dk, HV = m.H * m.dv;
    uint8_t* w = reinterpret_cast<uint8_t*>(m.workspace);
    auto carve = [&](size_t bytes) {
        uint8_t* p = w;
        w += (bytes + 255) & ~(size_t)255;
        return p;
    };
    __nv_bfloat16* q_rot = reinterpret_cast<__nv_bfloat16*>(carve(M * HK * 2));
    __nv_bfloat16* k_pr = reinterpret_cast<__nv_bfloat16*>(carve(M * HK * 2));
    __nv_bfloat16* v = reinterpret_cast<__nv_bfloat16*>(carve(M * HV * 2));
    __nv_bfloat16* g = reinterpret_cast<__nv_bfloat16*>(carve(M * HV * 2));
    float* y = reinterpret_cast<float*>(carve(M * HV * 4));
    float2* rot = reinterpret_cast<float2*>(carve((size_t)m.N * (m.dk / 2) * 8));
    if (m.xpos) {
        const long long n_cs = (long long)m.N * (m.dk / 2);
        k_rot_table<<<(int)((n_cs + 255) / 256), 256, 0, s>>>(rot, m.N, m.dk / 2, m.pos_offset, log2(m.theta_base));
        ret_status st0 = check_launch("ret_msr_forward: rotation table");
        if (st0 != RET_OK) return st0;
    }

    // 1. projections with the fused epilogue
    GemmSegment segs[4] = {{m.Wq, HK}, {m.Wk, HK}, {m.Wv, HV}, {m.Wg, HV}};
    GemmEpilogue epi;
    memset(&epi, 0, sizeof(epi));
    epi.seg[0] = {q_rot, HK, m.xpos ? kEpiRotate : kEpiStore, RET_BF16, 1.f, m.dk};
    epi.seg[1] = {k_pr, HK, kEpiRotateScaleZeta, RET_BF16, (float)m.k_scale, m.dk};
    epi.seg[2] = {v, HV, kEpiStore, RET_BF16, 1.f, m.dv};
    epi.seg[3] = {g, HV, kEpiSwish, RET_BF16, 1.f, m.dv};
    epi.seq = m.N;
    epi.chunk = m.chunk;
    epi.xpos = m.xpos;
    epi.pos_offset = m.pos_offset;
    epi.log2base = log2(m.theta_base);
    epi.rot_cs = m.xpos ? rot : nullptr;
    memcpy(epi.log2g, m.hc.log2g, sizeof(epi.log2g));
    ret_status st = launch_gemm(m.X, (int)M, m.dmodel, segs, 4, epi, s);
    if (st != RET_OK) return st;

    // 2. retention on the prepared q_rot, k', v; fp32 output
    RetArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q_rot; a.k = k_pr; a.v = v; a.out = y; a.final_state = nullptr;
    a.B = m.B; a.N = m.N; a.H = m.H; a.dk = m.dk; a.dv = m.dv; a.chunk = m.chunk;
    a.in_dt = RET_BF16; a.out_dt = RET_F32; a.xpos = 0; a.pos_offset = 0; a.theta_base = 10000.0;
    a.hc = m.hc;
    st = launch_chunkwise_main(a, q_rot, m.dk, k_pr, s);
    if (st != RET_OK) return st;

    // 3. GroupNorm per (token, head) times swish(G), written over swish(G)
    const int rows = (int)(M * m.H);
    const int blocks = (rows + 7) / 8;
    switch (m.dv / 32) {
        case 4: k_gn_gate<4><<<blocks, 256, 0, s>>>(y, g, rows, m.dv, (float)m.eps); break;
        case 8: k_gn_gate<8><<<blocks, 256, 0, s>>>(y, g, rows, m.dv, (float)m.eps); break;
        case 16: k_gn_gate<16><<<blocks, 256, 0, s>>>(y, g, rows, m.dv, (float)m.eps); break;
        case 32: k_gn_gate<32><<<blocks, 256, 0, s>>>(y, g, rows, m.dv, (float)m.eps); break;
        default: return fail(RET_ERR_UNSUPPORTED, "ret_msr_forward: d_v must be 128, 256, 512 or 1024");
    }
    st = check_launch("ret_msr_forward: group norm and gate");
    if (st != RET_OK) return st;

    // 4. output projection
    GemmSegment so[1] = {{m.Wo, m.dmodel}};
    GemmEpilogue eo;
    memset(&eo, 0, sizeof(eo));
    eo.seg[0] = {m.out, m.dmodel, m.residual ? kEpiResidual : kEpiStore, m.out_dt, 1.f, 0,
                 reinterpret_cast<const __nv_bfloat16*>(m.residual), m.dmodel};
    eo.seq = m.N;
    eo.chunk = m.chunk;
    return launch_gemm(g, (int)M, HV, so, 1, eo, s);
}

}  // namespace ret
