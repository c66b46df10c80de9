// k_chunk_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) chunkwise retention
// forward for bf16 inputs with fp32 accumulation and an fp32 carried state.
//
// Mathematics ("Hybrid Architectures: RetNet and the Three Computation
// Paradigms", section 7.2; RetNet paper summary, Eq. 7).  For a chunk of L
// rows starting at token n0 and 0-based rows r, c:
//     out_r = sum_{c<=r} gamma^(r-c) (q_r . k_c) v_c + gamma^(r+1) q_r^T R_prev
//     R     = gamma^L R_prev + sum_c gamma^(L-1-c) k_c v_c^T
// The kernel folds every decay factor into one scaled key and one row scale:
//     k'_c = gamma^(L-1-c) k_c                      (the state-update zeta)
//     T    = gamma^L R_prev                          (pre-scaled state)
//     out_r = gamma^(r+1-L) [ sum_{c<=r} (q_r . k'_c) v_c + q_r^T T ]
//     R     = T + K'^T V
// because gamma^(r-c) = gamma^(r+1-L) * gamma^(L-1-c) and gamma^(r+1) =
// gamma^(r+1-L) * gamma^L.  So the decay mask D becomes a plain causal mask
// on Q K'^T, generated in registers, and the intra-chunk scores, the cross
// read-out and the state update all feed one fp32 TMEM accumulator each.
// The row scale gamma^(r+1-L) is at most gamma^-(L-1), so the kernel takes
// heads with gamma^chunk >= 2^-60 (others go to the CUDA-core kernel).
//
// Work split: one CTA per (batch, head, 64-column tile of d_v), walking the
// chunks of its sequence in order.  Per chunk:
//   TMA     Q, K (d_k x chunk, 128-byte swizzled slabs) and the V tile
//   CUDA    rotate Q and K in place (xPos, consecutive pairs, one thread per
//           pair, incremental angle per row), scale K rows by zeta
//   tcgen05 A' = Q K'^T -> TMEM;  O' = Q T -> TMEM;  R += K'^T V -> TMEM
//   CUDA    P' = tril(A') as packed bf16 back into TMEM; T = gamma^L R to
//           TMEM (fp32) and to shared memory (bf16, next chunk's read-out)
//   tcgen05 O' += P' V   (A operand from TMEM)
//   CUDA    out = gamma^(r+1-L) O'  -> global
// TMEM columns: [0,128) A'/P', [128,192) O', [192, 192 + dk/2) R (two
// 128-row blocks for d_k = 256).
#include "kernels.h"
#include "tc_util.cuh"
#include "tmap.h"

namespace ret {

static __device__ int g_err_chunk_tc = 0;

cudaError_t read_clear_error_chunk_tc(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_err_chunk_tc, sizeof(int));
    if (e == cudaSuccess && *flag) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_err_chunk_tc, &zero, sizeof(int));
    }
    return e;
}

namespace {

constexpr int kC = 128;       // chunk rows handled by the kernel (M of every MMA)
constexpr int kW = 64;        // d_v columns per CTA
constexpr int kThreads = 128;
constexpr uint32_t kColA = 0, kColO = 128, kColS = 192;

struct TcParams {
    CUtensorMap tq, tk, tv;
    void* out;
    float* fstate;
    int N, H, dv;
    int xpos;
    long long pos0;
    double log2base;
    HeadConsts hc;
};

template <int DK>
struct Smem {
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + DK * kC * 2;
    static constexpr uint32_t kV = kK + DK * kC * 2;
    static constexpr uint32_t kT = kV + kC * kW * 2;
    static constexpr uint32_t kEnd = kT + DK * 128;
    static constexpr uint32_t kBytes = kEnd + 1024;  // + alignment slack
};

__device__ __forceinline__ bool all_ok(bool ok) { return __syncthreads_and(ok ? 1 : 0) != 0; }

template <int DK, typename Tout>
__global__ void __launch_bounds__(kThreads, 1) k_chunkwise_tc(const __grid_constant__ TcParams p) {
    constexpr int kSlabs = DK / 64;
    constexpr int kPairs = DK / 2;
    constexpr int kTpp = kThreads / kPairs;  // threads per rotation pair (1 or 2)
    constexpr int kMB = DK / 128;            // 128-row blocks of the state
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = sm + Smem<DK>::kQ;
    uint8_t* sK = sm + Smem<DK>::kK;
    uint8_t* sV = sm + Smem<DK>::kV;
    uint8_t* sT = sm + Smem<DK>::kT;
    __shared__ uint64_t bar_tma, bar_mma;
    __shared__ uint32_t s_tmem;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j0 = blockIdx.x * kW, h = blockIdx.y, b = blockIdx.z;
    const int N = p.N;
    const double lg = p.hc.log2g[h];

    if (tid == 0) {
        tc::mbar_init(&bar_tma, 1);
        tc::mbar_init(&bar_mma, 1);
        tc::fence_barrier_init();
        tc::prefetch_tmap(&p.tq);
        tc::prefetch_tmap(&p.tk);
        tc::prefetch_tmap(&p.tv);
    }
    if (warp == 0) tc::tmem_alloc(&s_tmem, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tb = s_tmem;
    const uint32_t lane_base = tb + ((uint32_t)(warp * 32) << 16);

    // rotation constants of this thread's pair
    const int pr = tid % kPairs, rsub = tid / kPairs;
    float wc = 1.f, ws = 0.f;  // e^{-i kTpp theta_p}
    double theta = 0.0;
    if (p.xpos) {
        theta = exp2(-2.0 * pr / DK * p.log2base);
        double sn, cs;
        sincos((double)kTpp * theta, &sn, &cs);
        wc = (float)cs;
        ws = (float)(-sn);
    }
    const float g_step = (float)exp2((double)kTpp * lg);  // gamma^kTpp
    const uint32_t slab_off = (uint32_t)(pr / 32) * (kC * 128);
    const uint32_t wl = pr % 32;

    const uint32_t idesc_qk = tc::idesc_bf16_f32(128, 128, 0, 0);
    const uint32_t idesc_qt = tc::idesc_bf16_f32(128, kW, 0, 1);
    const uint32_t idesc_st = tc::idesc_bf16_f32(128, kW, 1, 1);
    const uint32_t idesc_pv = tc::idesc_bf16_f32(128, kW, 0, 1);
    const uint32_t aQ = tc::smem_u32(sQ), aK = tc::smem_u32(sK), aV = tc::smem_u32(sV), aT = tc::smem_u32(sT);

    uint32_t ph_tma = 0, ph_mma = 0;
    bool ok = true;
    const int nchunks = (N + kC - 1) / kC;

    for (int jc = 0; jc < nchunks && ok; jc++) {
        const int n0 = jc * kC;
        const int L = min(kC, N - n0);
        const bool first = (jc == 0), last = (jc == nchunks - 1);

        // ---- TMA: Q, K slabs and the V tile of this chunk
        if (tid == 0) {
            tc::mbar_arrive_expect_tx(&bar_tma, 2 * DK * kC * 2 + kC * kW * 2);
            for (int s = 0; s < kSlabs; s++) {
                tc::tma_load_4d(sQ + s * kC * 128, &p.tq, &bar_tma, 64 * s, h, n0, b);
                tc::tma_load_4d(sK + s * kC * 128, &p.tk, &bar_tma, 64 * s, h, n0, b);
            }
            tc::tma_load_4d(sV, &p.tv, &bar_tma, j0, h, n0, b);
        }
        ok = all_ok(tc::mbar_wait(&bar_tma, ph_tma));
        ph_tma ^= 1;
        if (!ok) break;

        // ---- rotate Q and K in place; scale K rows by zeta_r = gamma^(L-1-r)
        {
            // this thread's rows: rsub, rsub + kTpp, ...; walk them downwards
            const int rtop = kC - kTpp + rsub;
            float zc = 1.f, zs = 0.f;
            if (p.xpos) {
                const double two_pi = 6.283185307179586476925286766559;
                double a = (double)(p.pos0 + n0 + rtop) * theta;
                a -= two_pi * rint(a / two_pi);
                double sn, cs;
                sincos(a, &sn, &cs);
                zc = (float)cs;
                zs = (float)sn;
            }
            // zeta_r = gamma^(L-1-r) for rows r < L; rows >= L are zero-filled by
            // the TMA load and get zeta 0.  r_first is this thread's largest row < L.
            const int r_first = (L - 1 >= rsub) ? rsub + kTpp * ((L - 1 - rsub) / kTpp) : -1;
            float zeta = 0.f;
            for (int r = rtop; r >= 0; r -= kTpp) {
                if (r == r_first) zeta = (float)exp2((double)(L - 1 - r) * lg);
                const uint32_t off = slab_off + tc::sw128_off((uint32_t)r, wl >> 2) + (wl & 3) * 4;
                if (p.xpos) {
                    uint32_t* qa = reinterpret_cast<uint32_t*>(sQ + off);
                    const uint32_t qw = *qa;
                    const float x0 = tc::bf16lo(qw), x1 = tc::bf16hi(qw);
                    *qa = tc::pack_bf16x2(x0 * zc - x1 * zs, x0 * zs + x1 * zc);
                }
                uint32_t* ka = reinterpret_cast<uint32_t*>(sK + off);
                const uint32_t kw = *ka;
                const float y0 = tc::bf16lo(kw), y1 = tc::bf16hi(kw);
                const float kc = zc * zeta, ks = zs * zeta;
                *ka = tc::pack_bf16x2(y0 * kc - y1 * ks, y0 * ks + y1 * kc);
                // step to row r - kTpp
                const float nc = zc * wc - zs * ws, ns = zc * ws + zs * wc;
                zc = nc;
                zs = ns;
                zeta *= g_step;
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        // ---- MMAs: A' = Q K'^T, O' = Q T (after the first chunk), R += K'^T V
        if (tid == 0) {
            for (int k = 0; k < DK / 16; k++) {
                const uint32_t off = (k / 4) * (kC * 128) + (k % 4) * 32;
                tc::mma_bf16_ss(tb + kColA, tc::sdesc_sw128(aQ + off, 16, 1024), tc::sdesc_sw128(aK + off, 16, 1024),
                                idesc_qk, k > 0);
            }
            if (!first) {
                for (int k = 0; k < DK / 16; k++) {
                    const uint32_t off = (k / 4) * (kC * 128) + (k % 4) * 32;
                    tc::mma_bf16_ss(tb + kColO, tc::sdesc_sw128(aQ + off, 16, 1024),
                                    tc::sdesc_sw128(aT + k * 2048, DK * 128, 1024), idesc_qt, k > 0);
                }
            }
            for (int mb = 0; mb < kMB; mb++) {
                for (int k = 0; k < kC / 16; k++) {
                    tc::mma_bf16_ss(tb + kColS + mb * kW,
                                    tc::sdesc_sw128(aK + mb * 2 * (kC * 128) + k * 2048, kC * 128, 1024),
                                    tc::sdesc_sw128(aV + k * 2048, kC * 128, 1024), idesc_st, (!first) || k > 0);
                }
            }
            tc::mma_commit(&bar_mma);
        }
        ok = all_ok(tc::mbar_wait(&bar_mma, ph_mma));
        ph_mma ^= 1;
        if (!ok) break;
        tc::tc_fence_after();

        // ---- P' = tril(A') as packed bf16 into TMEM columns [0, 64)
        {
            const int r = warp * 32 + lane;  // this thread's TMEM lane = query row
            uint32_t a[4][32];
#pragma unroll
            for (int q4 = 0; q4 < 4; q4++) tc::tmem_ld32(lane_base + kColA + 32 * q4, a[q4]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int half = 0; half < 2; half++) {
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int c = 64 * half + 2 * i;
                    const float lo = (c <= r) ? __uint_as_float(a[2 * half + (i >> 4)][(2 * i) & 31]) : 0.f;
                    const float hi = (c + 1 <= r) ? __uint_as_float(a[2 * half + (i >> 4)][(2 * i + 1) & 31]) : 0.f;
                    w[i] = tc::pack_bf16x2(lo, hi);
                }
                tc::tmem_st32(lane_base + kColA + 32 * half, w);
            }
        }
        // ---- T = gamma^L_next R  (TMEM fp32 in place, and bf16 to shared memory)
        if (!last) {
            const int Ln = min(kC, N - (n0 + kC));
            const float gL = (float)exp2((double)Ln * lg);
#pragma unroll
            for (int mb = 0; mb < kMB; mb++) {
                const int d = mb * 128 + warp * 32 + lane;  // state row
                uint32_t s[2][32];
                tc::tmem_ld32(lane_base + kColS + mb * kW, s[0]);
                tc::tmem_ld32(lane_base + kColS + mb * kW + 32, s[1]);
                tc::tmem_ld_wait();
#pragma unroll
                for (int hh = 0; hh < 2; hh++)
#pragma unroll
                    for (int i = 0; i < 32; i++) s[hh][i] = __float_as_uint(__uint_as_float(s[hh][i]) * gL);
                tc::tmem_st32(lane_base + kColS + mb * kW, s[0]);
                tc::tmem_st32(lane_base + kColS + mb * kW + 32, s[1]);
                // bf16 row d of T (MN-major: row = d, 64 columns = 128 bytes)
#pragma unroll
                for (int c16 = 0; c16 < 8; c16++) {
                    const int hh = c16 >> 2, base = (c16 & 3) * 8;
                    uint4 v;
                    v.x = tc::pack_bf16x2(__uint_as_float(s[hh][base + 0]), __uint_as_float(s[hh][base + 1]));
                    v.y = tc::pack_bf16x2(__uint_as_float(s[hh][base + 2]), __uint_as_float(s[hh][base + 3]));
                    v.z = tc::pack_bf16x2(__uint_as_float(s[hh][base + 4]), __uint_as_float(s[hh][base + 5]));
                    v.w = tc::pack_bf16x2(__uint_as_float(s[hh][base + 6]), __uint_as_float(s[hh][base + 7]));
                    *reinterpret_cast<uint4*>(sT + tc::sw128_off((uint32_t)d, (uint32_t)c16)) = v;
                }
            }
        }
        tc::tmem_st_wait();
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();

        // ---- O' += P' V   (A from TMEM)
        if (tid == 0) {
            for (int k = 0; k < kC / 16; k++)
                tc::mma_bf16_ts(tb + kColO, tb + kColA + 8 * k, tc::sdesc_sw128(aV + k * 2048, kC * 128, 1024),
                                idesc_pv, (!first) || k > 0);
            tc::mma_commit(&bar_mma);
        }
        ok = all_ok(tc::mbar_wait(&bar_mma, ph_mma));
        ph_mma ^= 1;
        if (!ok) break;
        tc::tc_fence_after();

        // ---- epilogue: out_r = gamma^(r+1-L) O'_r
        {
            const int r = warp * 32 + lane;
            uint32_t o[2][32];
            tc::tmem_ld32(lane_base + kColO, o[0]);
            tc::tmem_ld32(lane_base + kColO + 32, o[1]);
            tc::tmem_ld_wait();
            if (r < L) {
                const float sc = (float)exp2((double)(r + 1 - L) * lg);
                Tout* dst = reinterpret_cast<Tout*>(p.out) + (((size_t)b * N + n0 + r) * p.H + h) * p.dv + j0;
                if constexpr (sizeof(Tout) == 2) {
#pragma unroll
                    for (int c16 = 0; c16 < 8; c16++) {
                        const int hh = c16 >> 2, base = (c16 & 3) * 8;
                        uint4 v;
                        v.x = tc::pack_bf16x2(__uint_as_float(o[hh][base + 0]) * sc, __uint_as_float(o[hh][base + 1]) * sc);
                        v.y = tc::pack_bf16x2(__uint_as_float(o[hh][base + 2]) * sc, __uint_as_float(o[hh][base + 3]) * sc);
                        v.z = tc::pack_bf16x2(__uint_as_float(o[hh][base + 4]) * sc, __uint_as_float(o[hh][base + 5]) * sc);
                        v.w = tc::pack_bf16x2(__uint_as_float(o[hh][base + 6]) * sc, __uint_as_float(o[hh][base + 7]) * sc);
                        reinterpret_cast<uint4*>(dst)[c16] = v;
                    }
                } else {
#pragma unroll
                    for (int c4 = 0; c4 < 16; c4++) {
                        const int hh = c4 >> 3, base = (c4 & 7) * 4;
                        float4 v = make_float4(__uint_as_float(o[hh][base + 0]) * sc, __uint_as_float(o[hh][base + 1]) * sc,
                                               __uint_as_float(o[hh][base + 2]) * sc, __uint_as_float(o[hh][base + 3]) * sc);
                        reinterpret_cast<float4*>(dst)[c4] = v;
                    }
                }
            }
        }
        // ---- final state R after the last chunk
        if (last && p.fstate) {
#pragma unroll
            for (int mb = 0; mb < kMB; mb++) {
                const int d = mb * 128 + warp * 32 + lane;
                uint32_t s[2][32];
                tc::tmem_ld32(lane_base + kColS + mb * kW, s[0]);
                tc::tmem_ld32(lane_base + kColS + mb * kW + 32, s[1]);
                tc::tmem_ld_wait();
                float4* dst = reinterpret_cast<float4*>(p.fstate + (((size_t)b * p.H + h) * DK + d) * p.dv + j0);
#pragma unroll
                for (int c4 = 0; c4 < 16; c4++) {
                    const int hh = c4 >> 3, base = (c4 & 7) * 4;
                    dst[c4] = make_float4(__uint_as_float(s[hh][base]), __uint_as_float(s[hh][base + 1]),
                                          __uint_as_float(s[hh][base + 2]), __uint_as_float(s[hh][base + 3]));
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
    }

    if (!ok && tid == 0) atomicExch(&g_err_chunk_tc, kErrTimeout);
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tb, 512);
}

bool make_maps(const RetArgs& a, TcParams* p) {
    const uint64_t B = a.B, N = a.N, H = a.H, dk = a.dk, dv = a.dv;
    const uint64_t dq[4] = {dk, H, N, B};
    const uint64_t sq[3] = {dk * 2, H * dk * 2, N * H * dk * 2};
    const uint32_t bq[4] = {64, 1, (uint32_t)kC, 1};
    const uint64_t dvv[4] = {dv, H, N, B};
    const uint64_t svv[3] = {dv * 2, H * dv * 2, N * H * dv * 2};
    const uint32_t bv[4] = {64, 1, (uint32_t)kC, 1};
    return make_tmap_bf16(&p->tq, a.q, 4, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_tmap_bf16(&p->tk, a.k, 4, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_tmap_bf16(&p->tv, a.v, 4, dvv, svv, bv, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int DK, typename Tout>
ret_status launch_dk(const TcParams& p, const RetArgs& a, cudaStream_t s) {
    auto kern = k_chunkwise_tc<DK, Tout>;
    const int smem = (int)Smem<DK>::kBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return check_launch("chunkwise (tensor cores): smem attribute");
    dim3 grid(a.dv / kW, a.H, a.B);
    kern<<<grid, kThreads, smem, s>>>(p);
    return check_launch("chunkwise (tensor cores)");
}

}  // namespace

bool chunkwise_tc_supported(const RetArgs& a) {
    if (a.in_dt != RET_BF16) return false;
    if (a.chunk != kC || !(a.dk == 128 || a.dk == 256) || a.dv % kW != 0) return false;
    if (a.N > (1 << 30)) return false;
    for (int h = 0; h < a.H; h++)
        if (!(a.hc.log2g[h] * kC >= -60.0)) return false;
    return true;
}

ret_status launch_chunkwise_tc(const RetArgs& a, cudaStream_t s) {
    TcParams p;
    if (!make_maps(a, &p)) return RET_ERR_CUDA;
    p.out = a.out;
    p.fstate = a.final_state;
    p.N = a.N;
    p.H = a.H;
    p.dv = a.dv;
    p.xpos = a.xpos;
    p.pos0 = a.pos_offset;
    p.log2base = log2(a.theta_base);
    p.hc = a.hc;
    const bool f32 = a.out_dt == RET_F32;
    if (a.dk == 256) return f32 ? launch_dk<256, float>(p, a, s) : launch_dk<256, __nv_bfloat16>(p, a, s);
    return f32 ? launch_dk<128, float>(p, a, s) : launch_dk<128, __nv_bfloat16>(p, a, s);
}

}  // namespace ret
