// k_gemm.cu -- persistent warp-specialized tcgen05 GEMM, C = A B, for the
// MultiScaleRetention layer ("Hybrid Architectures: RetNet and the Three
// Computation Paradigms", section 9.1; RetNet paper summary, "Gated
// Multi-Scale Retention"): the four input projections X W_Q, X W_K, X W_V,
// X W_G in one launch with a fused epilogue, and the output projection Z W_O.
//
// A [M, K] bf16 row-major (K-major operand), B [K, N] bf16 row-major (the
// weight as stored, an MN-major operand).  Tiles 128 x 256 x 64, a 4-stage
// TMA ring (48 KB per stage), one tcgen05.mma issuer, two 256-column fp32
// accumulators in TMEM so that the epilogue of one tile overlaps the MMAs of
// the next, and two epilogue warpgroups (128 columns each).  The grid is
// persistent (one CTA per SM) and walks the tiles M-fastest.
//
// The B operand may be split into up to four column segments, each with its
// own tensor map and its own epilogue destination: that is how one launch
// computes [Q | K | V | G] = X [W_Q | W_K | W_V | W_G] without concatenating
// the weights.
#include "gemm.h"
#include "kernels.h"
#include "tc_util.cuh"
#include "tmap.h"

namespace ret {

static __device__ int g_err_gemm = 0;

cudaError_t read_clear_error_gemm(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_err_gemm, sizeof(int));
    if (e == cudaSuccess && *flag) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_err_gemm, &zero, sizeof(int));
    }
    return e;
}

namespace {

constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr int kABytes = BM * BK * 2;   // 16 KB
constexpr int kBBytes = BK * BN * 2;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 320;          // TMA warp, MMA warp, two epilogue warpgroups
constexpr int kSmemBytes = kStages * kStageBytes + 1024;

constexpr int kMaxRotPairs = 256;  // rotated head width up to 512

struct GemmParams {
    int rot_pairs;  // pairs of a rotated head (head_dim / 2), 0 without rotation
    CUtensorMap ta;
    CUtensorMap tb[4];
    int M, K;
    int nseg;
    int seg_n0[5];       // global column where segment s starts; seg_n0[nseg] = total N
    int tiles_n;         // N tiles over all segments
    int seg_tile0[5];    // first N tile of each segment
    GemmEpilogue epi;
};

struct GBars {
    uint64_t full[kStages], empty[kStages], accfull[2], accempty[2];
};

__device__ __forceinline__ void tile_coords(const GemmParams& p, int t, int& tm, int& tn, int& seg) {
    const int tiles_m = (p.M + BM - 1) / BM;
    tm = t % tiles_m;
    tn = t / tiles_m;
    seg = 0;
    while (seg + 1 < p.nseg && tn >= p.seg_tile0[seg + 1]) seg++;
}

// ------------------------------------------------------------ epilogues

__device__ __forceinline__ float swish(float x) { return x / (1.f + expf(-x)); }

// gelu(x) = x Phi(x) with the exact normal CDF, Phi(x) = (1 + erf(x / sqrt 2)) / 2.
__device__ __forceinline__ float gelu(float x) { return 0.5f * x * (1.f + erff(x * 0.70710678118654752f)); }

// Store 32 consecutive fp32 values of row m, starting at segment column c0.
// theta: the rotation frequencies theta_p of the rotated segments' heads,
// one per pair (shared memory, filled once per CTA).
__device__ __forceinline__ void epi_store(const GemmEpilogue& e, int seg, int m, int c0, const float (&v)[32],
                                          int ncols_valid, const double* theta) {
    const GemmSegOut& o = e.seg[seg];
    if (m >= e.M) return;
    if (o.kind == kEpiRotate || o.kind == kEpiRotateScaleZeta) {
        // xPos rotation of consecutive pairs within a head of width o.head_dim
        // at position pos_offset + (m % seq), then (keys) the scale and zeta
        // of the row's place in its chunk.
        const int n = m % e.seq;
        float w[32];
        float mult = 1.f;
        const int d0 = c0 % o.head_dim;
        const int hh = c0 / o.head_dim;
        if (o.kind == kEpiRotateScaleZeta) {
            const int r = n % e.chunk;
            const int L = min(e.chunk, e.seq - (n - r));
            // zeta = gamma^(L-1-r): the exponent in fp64, exp2 in fp32 (relative error ~1e-7)
            mult = o.scale * exp2f((float)((double)(L - 1 - r) * e.log2g[hh]));
        } else {
            mult = o.scale;
        }
        // (cos, sin) of the 16 pairs: from the per-call table, two pairs per
        // 16-byte load (the row's 16 pairs are 128 contiguous bytes, 128-byte
        // aligned since d0 is a multiple of 32), else evaluated here
        float csv[16], snv[16];
        if (e.xpos && e.rot_cs) {
            const float4* t4 = reinterpret_cast<const float4*>(e.rot_cs + (size_t)n * (o.head_dim >> 1) + (d0 >> 1));
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float4 t = __ldg(t4 + i);
                csv[2 * i] = t.x;
                snv[2 * i] = t.y;
                csv[2 * i + 1] = t.z;
                snv[2 * i + 1] = t.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; i++) {
                csv[i] = 1.f;
                snv[i] = 0.f;
                if (e.xpos) sincosf(rot_angle(e.pos_offset + n, theta[(d0 >> 1) + i]), &snv[i], &csv[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const float cs = csv[i] * mult, sn = snv[i] * mult;
            const float x0 = v[2 * i], x1 = v[2 * i + 1];
            w[2 * i] = x0 * cs - x1 * sn;
            w[2 * i + 1] = x0 * sn + x1 * cs;
        }
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(o.ptr) + (size_t)m * o.ld + c0;
#pragma unroll
        for (int c = 0; c < 4; c++) {
            uint4 u;
            u.x = tc::pack_bf16x2(w[8 * c + 0], w[8 * c + 1]);
            u.y = tc::pack_bf16x2(w[8 * c + 2], w[8 * c + 3]);
            u.z = tc::pack_bf16x2(w[8 * c + 4], w[8 * c + 5]);
            u.w = tc::pack_bf16x2(w[8 * c + 6], w[8 * c + 7]);
            reinterpret_cast<uint4*>(dst)[c] = u;
        }
        return;
    }
    float w[32];
    if (o.kind == kEpiSwish) {
#pragma unroll
        for (int i = 0; i < 32; i++) w[i] = swish(v[i]);
    } else if (o.kind == kEpiGelu) {
#pragma unroll
        for (int i = 0; i < 32; i++) w[i] = gelu(v[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 32; i++) w[i] = v[i] * o.scale;
    }
    if (o.kind == kEpiResidual) {
        const __nv_bfloat16* r = o.res + (size_t)m * o.res_ld + c0;
        if (ncols_valid >= 32) {
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const uint4 u = reinterpret_cast<const uint4*>(r)[c];
                const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const float2 f = __bfloat1622float2(hp[e]);
                    w[8 * c + 2 * e] += f.x;
                    w[8 * c + 2 * e + 1] += f.y;
                }
            }
        } else {
            for (int i = 0; i < ncols_valid; i++) w[i] += __bfloat162float(r[i]);
        }
    }
    if (o.dtype == RET_F32) {
        float* dst = reinterpret_cast<float*>(o.ptr) + (size_t)m * o.ld + c0;
        if (ncols_valid >= 32) {
#pragma unroll
            for (int c = 0; c < 8; c++)
                reinterpret_cast<float4*>(dst)[c] = make_float4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        } else {
            for (int i = 0; i < ncols_valid; i++) dst[i] = w[i];
        }
    } else {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(o.ptr) + (size_t)m * o.ld + c0;
        if (ncols_valid >= 32) {
#pragma unroll
            for (int c = 0; c < 4; c++) {
                uint4 u;
                u.x = tc::pack_bf16x2(w[8 * c + 0], w[8 * c + 1]);
                u.y = tc::pack_bf16x2(w[8 * c + 2], w[8 * c + 3]);
                u.z = tc::pack_bf16x2(w[8 * c + 4], w[8 * c + 5]);
                u.w = tc::pack_bf16x2(w[8 * c + 6], w[8 * c + 7]);
                reinterpret_cast<uint4*>(dst)[c] = u;
            }
        } else {
            for (int i = 0; i < ncols_valid; i++) dst[i] = __float2bfloat16_rn(w[i]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) k_gemm(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ GBars bars;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;
    __shared__ double s_theta[kMaxRotPairs];  // theta_p = base^(-2p/head_dim) of the rotated segments
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles_m = (p.M + BM - 1) / BM;
    const int ntiles = tiles_m * p.tiles_n;
    const int kblocks = (p.K + BK - 1) / BK;

    if (tid == 0) {
        for (int i = 0; i < kStages; i++) {
            tc::mbar_init(&bars.full[i], 1);
            tc::mbar_init(&bars.empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&bars.accfull[i], 1);
            tc::mbar_init(&bars.accempty[i], 8);
        }
        s_fail = 0;
        tc::fence_barrier_init();
        tc::prefetch_tmap(&p.ta);
        for (int s = 0; s < p.nseg; s++) tc::prefetch_tmap(&p.tb[s]);
    }
    if (warp == 1) tc::tmem_alloc(&s_tmem, 512);
    for (int i = tid; i < p.rot_pairs; i += kThreads) s_theta[i] = exp2(-2.0 * i / (2 * p.rot_pairs) * p.epi.log2base);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tbase = s_tmem;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;  // global k-block counter over this CTA's tiles
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                int tm, tn, seg;
                tile_coords(p, t, tm, tn, seg);
                const int ncol = (tn - p.seg_tile0[seg]) * BN;  // column within the segment
                for (int kb = 0; kb < kblocks && ok; kb++, it++) {
                    const int st = it % kStages, u = it / kStages;
                    if (u > 0) ok = tc::mbar_wait(&bars.empty[st], (u - 1) & 1);
                    if (!ok) break;
                    uint8_t* a = sm + st * kStageBytes;
                    uint8_t* b = a + kABytes;
                    tc::mbar_arrive_expect_tx(&bars.full[st], kStageBytes);
                    tc::tma_load_2d(a, &p.ta, &bars.full[st], kb * BK, tm * BM);
                    for (int nb = 0; nb < BN / 64; nb++)
                        tc::tma_load_2d(b + nb * (BK * 128), &p.tb[seg], &bars.full[st], ncol + 64 * nb, kb * BK);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(BM, BN, 0, 1);
            int it = 0, tl = 0;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, tl++) {
                const int ab = tl & 1;
                if (tl >= 2) ok = tc::mbar_wait(&bars.accempty[ab], ((tl >> 1) & 1) ^ 1);
                if (!ok) break;
                tc::tc_fence_after();
                const uint32_t d = tbase + 256 * ab;
                for (int kb = 0; kb < kblocks && ok; kb++, it++) {
                    const int st = it % kStages, u = it / kStages;
                    ok = tc::mbar_wait(&bars.full[st], u & 1);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const uint32_t a = tc::smem_u32(sm + st * kStageBytes);
                    const uint32_t b = a + kABytes;
                    for (int k = 0; k < BK / 16; k++)
                        tc::mma_bf16_ss(d, tc::sdesc_sw128(a + k * 32, 16, 1024),
                                        tc::sdesc_sw128(b + k * 2048, BK * 128, 1024), idesc, (kb > 0) || (k > 0));
                    tc::mma_commit(&bars.empty[st]);
                }
                tc::mma_commit(&bars.accfull[ab]);
            }
        }
    } else {
        const int quarter = warp & 3, wg = (warp - 2) >> 2;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        int tl = 0;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, tl++) {
            int tm, tn, seg;
            tile_coords(p, t, tm, tn, seg);
            const int ab = tl & 1;
            ok = tc::mbar_wait(&bars.accfull[ab], (tl >> 1) & 1);
            if (!ok) break;
            tc::tc_fence_after();
            const int m = tm * BM + quarter * 32 + lane;
            const int seg_cols = p.seg_n0[seg + 1] - p.seg_n0[seg];
            for (int c = 0; c < 4; c++) {
                const int col = 128 * wg + 32 * c;
                uint32_t r[32];
                tc::tmem_ld32(tbase + lane_off + 256 * ab + col, r);
                tc::tmem_ld_wait();
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
                const int c0 = (tn - p.seg_tile0[seg]) * BN + col;  // column within the segment
                if (c0 < seg_cols) epi_store(p.epi, seg, m, c0, v, seg_cols - c0, s_theta);
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars.accempty[ab]);
        }
    }
    if (!ok) atomicExch(&s_fail, 1);
    tc::tc_fence_before();
    __syncthreads();
    if (s_fail && tid == 0) atomicExch(&g_err_gemm, kErrTimeout);
    if (warp == 1) tc::tmem_dealloc(tbase, 512);
}

}  // namespace

ret_status launch_gemm(const void* A, int M, int K, const GemmSegment* segs, int nseg, const GemmEpilogue& epi,
                       cudaStream_t s) {
    if (nseg < 1 || nseg > 4) return fail(RET_ERR_INVALID_ARG, "gemm: 1..4 segments");
    GemmParams p;
    memset(&p, 0, sizeof(p));
    const uint64_t da[2] = {(uint64_t)K, (uint64_t)M};
    const uint64_t sa[1] = {(uint64_t)K * 2};
    const uint32_t ba[2] = {BK, BM};
    if (!make_tmap_bf16(&p.ta, A, 2, da, sa, ba, CU_TENSOR_MAP_SWIZZLE_128B)) return RET_ERR_CUDA;
    p.M = M;
    p.K = K;
    p.nseg = nseg;
    int n0 = 0, t0 = 0;
    for (int i = 0; i < nseg; i++) {
        const uint64_t db[2] = {(uint64_t)segs[i].N, (uint64_t)K};
        const uint64_t sb[1] = {(uint64_t)segs[i].N * 2};
        const uint32_t bb[2] = {64, BK};
        if (!make_tmap_bf16(&p.tb[i], segs[i].B, 2, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_128B)) return RET_ERR_CUDA;
        p.seg_n0[i] = n0;
        p.seg_tile0[i] = t0;
        n0 += segs[i].N;
        t0 += (segs[i].N + BN - 1) / BN;
    }
    p.seg_n0[nseg] = n0;
    p.seg_tile0[nseg] = t0;
    p.tiles_n = t0;
    p.epi = epi;
    p.epi.M = M;
    p.rot_pairs = 0;
    for (int i = 0; i < nseg; i++) {
        const GemmSegOut& o = epi.seg[i];
        if (epi.xpos && (o.kind == kEpiRotate || o.kind == kEpiRotateScaleZeta)) {
            if (o.head_dim < 2 || o.head_dim / 2 > kMaxRotPairs || (p.rot_pairs && p.rot_pairs != o.head_dim / 2))
                return fail(RET_ERR_UNSUPPORTED, "gemm: rotated heads of different widths or wider than 512");
            p.rot_pairs = o.head_dim / 2;
        }
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int ntiles = ((M + BM - 1) / BM) * t0;
    const int grid = ntiles < sms ? ntiles : sms;
    if (cudaFuncSetAttribute(k_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
        return check_launch("gemm: smem attribute");
    k_gemm<<<grid, kThreads, kSmemBytes, s>>>(p);
    return check_launch("gemm");
}

ret_status launch_linear(const void* X, const void* W, void* Y, int M, int N, int K, ret_dtype out_dt,
                         cudaStream_t s) {
    GemmSegment seg[1] = {{W, N}};
    GemmEpilogue e;
    memset(&e, 0, sizeof(e));
    e.seg[0] = {Y, N, kEpiStore, out_dt, 1.f, 0, nullptr, 0};
    e.seq = 1;
    e.chunk = 1;
    return launch_gemm(X, M, K, seg, 1, e, s);
}

}  // namespace ret
