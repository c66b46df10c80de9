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
// the next, and two epilogue warpgroups (128 columns each) that stage each
// 128-row output box in shared memory and store it with one TMA store.  The
// grid is persistent (one CTA per SM) and walks the tiles M-fastest.
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
// Output staging: per epilogue warpgroup one 128-row box of 128-byte rows
// (64 bf16 or 32 fp32 columns) in the TMA's 128-byte swizzle.
constexpr int kOutBoxBytes = BM * 128;   // 16 KB
constexpr int kSmemBytes = kStages * kStageBytes + 2 * kOutBoxBytes + 1024;

struct GemmParams {
    CUtensorMap ta;
    CUtensorMap tb[4];
    CUtensorMap to[4];   // each segment's output [M, N_seg], box 128 rows x 128 bytes
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

// The 32 epilogue values of row m at segment column c0 (ncols_valid of them
// inside the segment; the rest, and rows past M, are zero).  Rotations use
// the per-call (cos, sin) table, two pairs per 16-byte load (a row's 16
// pairs are 128 contiguous bytes, 128-byte aligned since c0 is a multiple of
// 32 within its head).
__device__ __forceinline__ void epi_values(const GemmEpilogue& e, int seg, int m, int c0, const float (&v)[32],
                                           int ncols_valid, float (&w)[32]) {
    const GemmSegOut& o = e.seg[seg];
    if (m >= e.M) {
#pragma unroll
        for (int i = 0; i < 32; i++) w[i] = 0.f;
        return;
    }
    if (o.kind == kEpiRotate || o.kind == kEpiRotateScaleZeta) {
        // xPos rotation of consecutive pairs within a head of width o.head_dim
        // at position pos_offset + (m % seq), then (keys) the scale and zeta
        // of the row's place in its chunk.
        const int n = m % e.seq;
        float mult = o.scale;
        const int d0 = c0 % o.head_dim;
        const int hh = c0 / o.head_dim;
        if (o.kind == kEpiRotateScaleZeta) {
            const int r = n % e.chunk;
            const int L = min(e.chunk, e.seq - (n - r));
            // zeta = gamma^(L-1-r): the exponent in fp64, exp2 in fp32 (relative error ~1e-7)
            mult = o.scale * exp2f((float)((double)(L - 1 - r) * e.log2g[hh]));
        }
        float csv[16], snv[16];
        if (e.xpos) {
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
            }
        }
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const float cs = csv[i] * mult, sn = snv[i] * mult;
            const float x0 = v[2 * i], x1 = v[2 * i + 1];
            w[2 * i] = x0 * cs - x1 * sn;
            w[2 * i + 1] = x0 * sn + x1 * cs;
        }
    } else if (o.kind == kEpiSwish) {
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
                for (int e2 = 0; e2 < 4; e2++) {
                    const float2 f = __bfloat1622float2(hp[e2]);
                    w[8 * c + 2 * e2] += f.x;
                    w[8 * c + 2 * e2 + 1] += f.y;
                }
            }
        } else {
            for (int i = 0; i < ncols_valid; i++) w[i] += __bfloat162float(r[i]);
        }
    }
    if (ncols_valid < 32)
#pragma unroll
        for (int i = 0; i < 32; i++)
            if (i >= ncols_valid) w[i] = 0.f;
}

// Named barrier of one epilogue warpgroup (ids 1 and 2; 0 is __syncthreads),
// and the same barrier returning whether x holds in all 128 threads.
__device__ __forceinline__ void wg_sync(int wg) { asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory"); }
__device__ __forceinline__ bool wg_all(int wg, bool x) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)x), "r"(1 + wg)
        : "memory");
    return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1) k_gemm(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ GBars bars;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;
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
        // Epilogue warpgroups: warps 2-5 and 6-9, each on TMEM lanes 0..127
        // (a warp reaches the lane quarter warp % 4), one 128-column half of
        // the accumulator each.  Every 32 columns: TMEM -> registers, the
        // segment's epilogue, then the values into the warpgroup's staging
        // box (128 rows of 128 bytes: 64 bf16 or 32 fp32 columns, 128-byte
        // swizzle); a full box goes out in one TMA store (rows past M and
        // columns past the segment are clipped by the TMA).  The warpgroup
        // agrees on every wait's outcome before any of its barriers, so a
        // timed-out wait cannot leave part of it at a barrier.
        const int quarter = warp & 3, wg = (warp - 2) >> 2;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool leader = warp == 2 + 4 * wg && lane == 0;  // issues the warpgroup's stores
        uint8_t* box = sm + kStages * kStageBytes + wg * kOutBoxBytes;
        const uint32_t r = (uint32_t)(quarter * 32 + lane);   // row in the tile
        int tl = 0;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, tl++) {
            int tm, tn, seg;
            tile_coords(p, t, tm, tn, seg);
            const int ab = tl & 1;
            ok = wg_all(wg, tc::mbar_wait(&bars.accfull[ab], (tl >> 1) & 1));
            if (!ok) break;
            tc::tc_fence_after();
            const int m = tm * BM + (int)r;
            const int seg_cols = p.seg_n0[seg + 1] - p.seg_n0[seg];
            const bool f32 = p.epi.seg[seg].dtype == RET_F32;
            for (int c = 0; c < 4; c++) {
                const int col = 128 * wg + 32 * c;
                uint32_t rr[32];
                tc::tmem_ld32(tbase + lane_off + 256 * ab + col, rr);
                tc::tmem_ld_wait();
                float v[32], w[32];
#pragma unroll
                for (int i = 0; i < 32; i++) v[i] = __uint_as_float(rr[i]);
                const int c0 = (tn - p.seg_tile0[seg]) * BN + col;  // column within the segment
                if (c0 < seg_cols) {
                    epi_values(p.epi, seg, m, c0, v, seg_cols - c0, w);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i++) w[i] = 0.f;
                }
                // a box starts at every chunk (fp32) or every even chunk (bf16)
                const bool first = f32 || (c & 1) == 0, last = f32 || (c & 1) == 1;
                if (first) {
                    if (leader) tc::bulk_wait_group_read<0>();  // the previous box has been read
                    wg_sync(wg);
                }
                if (f32) {
#pragma unroll
                    for (int c4 = 0; c4 < 8; c4++)
                        *reinterpret_cast<float4*>(box + tc::sw128_off(r, (uint32_t)c4)) =
                            make_float4(w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
                } else {
                    const uint32_t h = (uint32_t)(c & 1);  // half of the 128-byte row
#pragma unroll
                    for (int c16 = 0; c16 < 4; c16++) {
                        uint4 u;
                        u.x = tc::pack_bf16x2(w[8 * c16 + 0], w[8 * c16 + 1]);
                        u.y = tc::pack_bf16x2(w[8 * c16 + 2], w[8 * c16 + 3]);
                        u.z = tc::pack_bf16x2(w[8 * c16 + 4], w[8 * c16 + 5]);
                        u.w = tc::pack_bf16x2(w[8 * c16 + 6], w[8 * c16 + 7]);
                        *reinterpret_cast<uint4*>(box + tc::sw128_off(r, 4 * h + (uint32_t)c16)) = u;
                    }
                }
                if (last) {
                    tc::fence_proxy_async_smem();
                    wg_sync(wg);
                    const int x0 = f32 ? c0 : c0 - 32;  // the box's first column
                    if (leader && x0 < seg_cols) {
                        tc::tma_store_2d(&p.to[seg], box, x0, tm * BM);
                        tc::bulk_commit_group();
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars.accempty[ab]);
        }
        if (leader) tc::bulk_wait_group<0>();  // every box is in global memory
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
    for (int i = 0; i < nseg; i++) {
        const GemmSegOut& o = epi.seg[i];
        if (epi.xpos && (o.kind == kEpiRotate || o.kind == kEpiRotateScaleZeta) &&
            (!epi.rot_cs || o.head_dim < 32 || o.head_dim % 32))
            return fail(RET_ERR_UNSUPPORTED, "gemm: rotated heads need the (cos, sin) table and a width multiple of 32");
        // output map: [M, N_seg] with row pitch ld, box 128 rows x 128 bytes
        const bool f32 = o.dtype == RET_F32;
        const uint64_t dout[2] = {(uint64_t)segs[i].N, (uint64_t)M};
        const uint64_t sout[1] = {(uint64_t)o.ld * (f32 ? 4 : 2)};
        const uint32_t bout[2] = {f32 ? 32u : 64u, (uint32_t)BM};
        if (!(f32 ? make_tmap_f32 : make_tmap_bf16)(&p.to[i], o.ptr, 2, dout, sout, bout, CU_TENSOR_MAP_SWIZZLE_128B))
            return RET_ERR_CUDA;
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
