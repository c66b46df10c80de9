// k_simt.cu -- CUDA-core kernels:
//   * xPos rotation in place ("Hybrid Architectures: RetNet and the Three
//     Computation Paradigms", sections 6.6 and 6.8);
//   * fp32 chunkwise forward (same page, section 7.2) -- the fp32 path and
//     the fallback for shapes the tensor-core kernel does not take;
//   * parallel form (section 4.3) and recurrent form (section 2.1), used to
//     cross-check the chunkwise path on the device.
// All arithmetic is fp32 FFMA (no TF32); decay powers are evaluated in fp64
// and rounded once.
#include <algorithm>

#include "kernels.h"

namespace ret {

// ----------------------------------------------------------------- rotation

template <typename T>
__global__ void k_xpos_rotate(T* __restrict__ x, int N, int H, int d, size_t total_pairs,
                              long long pos_offset, double log2base, float sign) {
    extern __shared__ double s_theta[];
    const int half = d / 2;
    for (int p = threadIdx.x; p < half; p += blockDim.x) s_theta[p] = exp2(-2.0 * p / d * log2base);
    __syncthreads();
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total_pairs;
         i += (size_t)gridDim.x * blockDim.x) {
        const int p = (int)(i % half);
        const size_t row = i / half;  // ((b * N + n) * H + h)
        const int n = (int)((row / H) % N);
        float sn, cs;
        sincosf(rot_angle(pos_offset + n, s_theta[p]), &sn, &cs);
        sn *= sign;  // -1: the inverse (transposed) rotation
        const size_t e = row * d + 2 * p;
        const float x0 = ld_as_float(x, e), x1 = ld_as_float(x, e + 1);
        st_from_float(x, e, x0 * cs - x1 * sn);
        st_from_float(x, e + 1, x0 * sn + x1 * cs);
    }
}

ret_status launch_xpos_rotate(void* x, ret_dtype dt, int B, int N, int H, int d, long long pos_offset,
                              double theta_base, cudaStream_t s, bool inverse) {
    const size_t total = (size_t)B * N * H * (d / 2);
    const int threads = 256;
    const int blocks = (int)std::min<size_t>((total + threads - 1) / threads, 148 * 16);
    const size_t smem = (size_t)(d / 2) * sizeof(double);
    if (smem > 48 * 1024) return fail(RET_ERR_UNSUPPORTED, "ret_xpos_rotate: d too large");
    const double lb = log2(theta_base);
    if (dt == RET_BF16)
        k_xpos_rotate<<<blocks, threads, smem, s>>>((__nv_bfloat16*)x, N, H, d, total, pos_offset, lb,
                                                    inverse ? -1.f : 1.f);
    else
        k_xpos_rotate<<<blocks, threads, smem, s>>>((float*)x, N, H, d, total, pos_offset, lb, inverse ? -1.f : 1.f);
    return check_launch("ret_xpos_rotate");
}

// Load row `n` of a [B, N, H, d] tensor (head h, batch b) into dst[0..d) as
// fp32, rotated by position pos when xpos is set.  Called by a whole block.
template <typename T>
__device__ __forceinline__ void load_rows_rotated(const T* __restrict__ src, int b, int n0, int rows, int N,
                                                  int H, int h, int d, float* dst, int ld, bool xpos,
                                                  long long pos0, const double* theta) {
    if (xpos) {
        const int half = d / 2;
        for (int idx = threadIdx.x; idx < rows * half; idx += blockDim.x) {
            const int r = idx / half, p = idx % half;
            const size_t e = (((size_t)b * N + n0 + r) * H + h) * d + 2 * p;
            const float x0 = ld_as_float(src, e), x1 = ld_as_float(src, e + 1);
            float sn, cs;
            sincosf(rot_angle(pos0 + n0 + r, theta[p]), &sn, &cs);
            dst[r * ld + 2 * p] = x0 * cs - x1 * sn;
            dst[r * ld + 2 * p + 1] = x0 * sn + x1 * cs;
        }
    } else {
        for (int idx = threadIdx.x; idx < rows * d; idx += blockDim.x) {
            const int r = idx / d, c = idx % d;
            dst[r * ld + c] = ld_as_float(src, (((size_t)b * N + n0 + r) * H + h) * d + c);
        }
    }
}

// ------------------------------------------------------ fp32 chunkwise form
//
// One block per (dv tile, head, batch); the chunks of the sequence are walked
// in order with the state R (dk x W) in shared memory.  Per chunk of L rows:
//   A[r][c] = gamma^(r-c) (q_r . k_c)  for c <= r, else 0      (Q K^T (.) D)
//   out_r   = sum_c A[r][c] v_c + gamma^(r+1) q_r^T R          (inner + cross)
//   R       = gamma^L R + sum_c gamma^(L-1-c) k_c v_c^T        (state update)

struct SimtChunkLayout {
    int W, ldk;
    size_t bytes;
};

// R: rows of q, k, v held at once (the chunk, or the whole sequence).
static SimtChunkLayout simt_chunk_layout(int C, int dk, int W, int R) {
    SimtChunkLayout l;
    l.W = W;
    l.ldk = dk + 1;
    size_t floats = (size_t)2 * R * l.ldk + (size_t)R * W + (size_t)C * (C + 1) + (size_t)dk * W + (C + 2);
    floats = (floats + 1) & ~(size_t)1;  // 8-byte alignment for the theta table
    l.bytes = floats * sizeof(float) + (size_t)(dk / 2 + 1) * sizeof(double);
    return l;
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_chunkwise_simt(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                        const Tin* __restrict__ v, HeadConsts hc, int N, int H,
                                                        int dk, int dv, int C, int W, Tout* __restrict__ out,
                                                        float* __restrict__ fstate, int xpos, long long pos0,
                                                        double log2base, int whole) {
    // whole: the sequence is short enough that all its rows of q, k, v are
    // loaded into shared memory once, before the chunk loop
    const int h = blockIdx.y, b = blockIdx.z, j0 = blockIdx.x * W;
    const int wt = min(W, dv - j0);
    const int ldk = dk + 1;
    const int RR = whole ? N : C;  // rows the buffers hold
    extern __shared__ float sm[];
    float* Qb = sm;
    float* Kb = Qb + (size_t)RR * ldk;
    float* Vb = Kb + (size_t)RR * ldk;
    float* As = Vb + (size_t)RR * W;
    float* Ss = As + (size_t)C * (C + 1);
    float* pw = Ss + (size_t)dk * W;
    size_t off = (size_t)2 * RR * ldk + (size_t)RR * W + (size_t)C * (C + 1) + (size_t)dk * W + (C + 2);
    off = (off + 1) & ~(size_t)1;
    double* theta = reinterpret_cast<double*>(sm + off);

    const double lg = hc.log2g[h];
    for (int e = threadIdx.x; e <= C; e += blockDim.x) pw[e] = gamma_pow_d(lg, e);
    for (int p = threadIdx.x; p < dk / 2; p += blockDim.x) theta[p] = exp2(-2.0 * p / dk * log2base);
    for (int e = threadIdx.x; e < dk * W; e += blockDim.x) Ss[e] = 0.f;
    __syncthreads();

    auto load = [&](int n0, int rows, float* Qd, float* Kd, float* Vd) {
        load_rows_rotated(q, b, n0, rows, N, H, h, dk, Qd, ldk, xpos != 0, pos0, theta);
        load_rows_rotated(k, b, n0, rows, N, H, h, dk, Kd, ldk, xpos != 0, pos0, theta);
        for (int idx = threadIdx.x; idx < rows * wt; idx += blockDim.x) {
            const int r = idx / wt, j = idx % wt;
            Vd[r * W + j] = ld_as_float(v, (((size_t)b * N + n0 + r) * H + h) * dv + j0 + j);
        }
    };
    if (whole) load(0, N, Qb, Kb, Vb);
    for (int c0 = 0; c0 < N; c0 += C) {
        const int L = min(C, N - c0);
        float* Qs = whole ? Qb + (size_t)c0 * ldk : Qb;
        float* Ks = whole ? Kb + (size_t)c0 * ldk : Kb;
        float* Vs = whole ? Vb + (size_t)c0 * W : Vb;
        if (!whole) load(c0, L, Qs, Ks, Vs);
        __syncthreads();
        for (int idx = threadIdx.x; idx < L * L; idx += blockDim.x) {
            const int r = idx / L, c = idx % L;
            float a = 0.f;
            if (c <= r) {
                const float* qr = Qs + r * ldk;
                const float* kc = Ks + c * ldk;
                for (int d = 0; d < dk; d++) a = fmaf(qr[d], kc[d], a);
                a *= pw[r - c];
            }
            As[r * (C + 1) + c] = a;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < L * wt; idx += blockDim.x) {
            const int r = idx / wt, j = idx % wt;
            float inner = 0.f, cross = 0.f;
            for (int c = 0; c <= r; c++) inner = fmaf(As[r * (C + 1) + c], Vs[c * W + j], inner);
            const float* qr = Qs + r * ldk;
            for (int d = 0; d < dk; d++) cross = fmaf(qr[d], Ss[d * W + j], cross);
            st_from_float(out, (((size_t)b * N + c0 + r) * H + h) * dv + j0 + j, fmaf(pw[r + 1], cross, inner));
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < dk * wt; idx += blockDim.x) {
            const int d = idx / wt, j = idx % wt;
            float acc = 0.f;
            for (int c = 0; c < L; c++) acc = fmaf(pw[L - 1 - c] * Ks[c * ldk + d], Vs[c * W + j], acc);
            Ss[d * W + j] = fmaf(pw[L], Ss[d * W + j], acc);
        }
        __syncthreads();
    }
    if (fstate) {
        for (int idx = threadIdx.x; idx < dk * wt; idx += blockDim.x) {
            const int d = idx / wt, j = idx % wt;
            fstate[(((size_t)b * H + h) * dk + d) * dv + j0 + j] = Ss[d * W + j];
        }
    }
}

ret_status launch_chunkwise_simt(const RetArgs& a, cudaStream_t s) {
    const int C = std::min(a.chunk, a.N);
    SimtChunkLayout lay{};
    int W = 0;
    for (int w : {64, 32, 16, 8}) {
        if (w > a.dv && w != 8) continue;
        lay = simt_chunk_layout(C, a.dk, w, C);
        if (lay.bytes <= 200 * 1024) { W = w; break; }
    }
    // a short sequence is loaded once (one round of global-load latency
    // instead of one per chunk)
    int whole = 0;
    if (W != 0 && a.N > C) {
        const SimtChunkLayout lw = simt_chunk_layout(C, a.dk, W, a.N);
        if (lw.bytes <= 64 * 1024) {
            lay = lw;
            whole = 1;
        }
    }
    if (W == 0)
        return fail(RET_ERR_UNSUPPORTED, "chunkwise (CUDA-core path): chunk=%d dk=%d does not fit shared memory",
                    a.chunk, a.dk);
    dim3 grid((a.dv + W - 1) / W, a.H, a.B);
    const double lb = log2(a.theta_base);
#define RET_LAUNCH_SIMT(TI, TO)                                                                               \
    do {                                                                                                      \
        auto kern = k_chunkwise_simt<TI, TO>;                                                                 \
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.bytes) !=        \
            cudaSuccess)                                                                                      \
            return check_launch("chunkwise (CUDA-core path): smem attribute");                               \
        kern<<<grid, 256, lay.bytes, s>>>((const TI*)a.q, (const TI*)a.k, (const TI*)a.v, a.hc, a.N, a.H,    \
                                          a.dk, a.dv, C, W, (TO*)a.out, a.final_state, a.xpos, a.pos_offset, \
                                          lb, whole);                                                         \
    } while (0)
    if (a.in_dt == RET_F32 && a.out_dt == RET_F32) RET_LAUNCH_SIMT(float, float);
    else if (a.in_dt == RET_F32) RET_LAUNCH_SIMT(float, __nv_bfloat16);
    else if (a.out_dt == RET_F32) RET_LAUNCH_SIMT(__nv_bfloat16, float);
    else RET_LAUNCH_SIMT(__nv_bfloat16, __nv_bfloat16);
#undef RET_LAUNCH_SIMT
    return check_launch("chunkwise (CUDA-core path)");
}

// ------------------------------------------------------------ parallel form
//
// out = (Q K^T (.) D) V with D_nm = gamma^(n-m) (n >= m).  One block per
// (query tile of 32 rows, dv tile of 64, batch-head); key tiles of 32 rows up
// to the diagonal.

constexpr int PQ = 32, PK = 32, PW = 64;

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_parallel_simt(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                       const Tin* __restrict__ v, HeadConsts hc, int N, int H,
                                                       int dk, int dv, Tout* __restrict__ out, int xpos,
                                                       long long pos0, double log2base) {
    const int q0 = blockIdx.x * PQ, j0 = blockIdx.y * PW;
    const int b = blockIdx.z / H, h = blockIdx.z % H;
    const int ldk = dk + 1;
    extern __shared__ double smd[];
    double* theta = smd;
    float* Qs = reinterpret_cast<float*>(smd + (dk / 2 + 1));
    float* Ks = Qs + PQ * ldk;
    float* Vs = Ks + PK * ldk;
    float* Ps = Vs + PK * PW;
    for (int p = threadIdx.x; p < dk / 2; p += blockDim.x) theta[p] = exp2(-2.0 * p / dk * log2base);
    __syncthreads();
    const int rq = min(PQ, N - q0);
    load_rows_rotated(q, b, q0, rq, N, H, h, dk, Qs, ldk, xpos != 0, pos0, theta);
    const double lg = hc.log2g[h];
    const int tj = threadIdx.x % PW, tr = threadIdx.x / PW;  // 4 row groups
    float acc[PQ / 4];
#pragma unroll
    for (int i = 0; i < PQ / 4; i++) acc[i] = 0.f;
    for (int k0 = 0; k0 < q0 + rq; k0 += PK) {
        const int rk = min(PK, N - k0);
        __syncthreads();
        load_rows_rotated(k, b, k0, rk, N, H, h, dk, Ks, ldk, xpos != 0, pos0, theta);
        for (int idx = threadIdx.x; idx < rk * PW; idx += blockDim.x) {
            const int r = idx / PW, j = idx % PW;
            Vs[r * PW + j] = (j0 + j < dv) ? ld_as_float(v, (((size_t)b * N + k0 + r) * H + h) * dv + j0 + j) : 0.f;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < PQ * PK; idx += blockDim.x) {
            const int r = idx / PK, c = idx % PK;
            const int n = q0 + r, m = k0 + c;
            float sc = 0.f;
            if (r < rq && c < rk && m <= n) {
                for (int d = 0; d < dk; d++) sc = fmaf(Qs[r * ldk + d], Ks[c * ldk + d], sc);
                sc *= gamma_pow_d(lg, n - m);
            }
            Ps[r * (PK + 1) + c] = sc;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < PQ / 4; i++) {
            const int r = tr + 4 * i;
            float a2 = acc[i];
            for (int c = 0; c < rk; c++) a2 = fmaf(Ps[r * (PK + 1) + c], Vs[c * PW + tj], a2);
            acc[i] = a2;
        }
    }
    if (j0 + tj < dv) {
#pragma unroll
        for (int i = 0; i < PQ / 4; i++) {
            const int r = tr + 4 * i;
            if (r < rq) st_from_float(out, (((size_t)b * N + q0 + r) * H + h) * dv + j0 + tj, acc[i]);
        }
    }
}

ret_status launch_parallel_simt(const RetArgs& a, cudaStream_t s) {
    if (a.dk > 256) return fail(RET_ERR_UNSUPPORTED, "ret_forward_parallel: dk > 256");
    const size_t bytes = (size_t)(a.dk / 2 + 1) * sizeof(double) +
                         ((size_t)(PQ + PK) * (a.dk + 1) + PK * PW + PQ * (PK + 1)) * sizeof(float);
    dim3 grid((a.N + PQ - 1) / PQ, (a.dv + PW - 1) / PW, a.B * a.H);
    const double lb = log2(a.theta_base);
#define RET_LAUNCH_PAR(TI, TO)                                                                                \
    do {                                                                                                      \
        auto kern = k_parallel_simt<TI, TO>;                                                                  \
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) \
            return check_launch("ret_forward_parallel: smem attribute");                                     \
        kern<<<grid, 256, bytes, s>>>((const TI*)a.q, (const TI*)a.k, (const TI*)a.v, a.hc, a.N, a.H, a.dk,  \
                                      a.dv, (TO*)a.out, a.xpos, a.pos_offset, lb);                            \
    } while (0)
    if (a.in_dt == RET_F32 && a.out_dt == RET_F32) RET_LAUNCH_PAR(float, float);
    else if (a.in_dt == RET_F32) RET_LAUNCH_PAR(float, __nv_bfloat16);
    else if (a.out_dt == RET_F32) RET_LAUNCH_PAR(__nv_bfloat16, float);
    else RET_LAUNCH_PAR(__nv_bfloat16, __nv_bfloat16);
#undef RET_LAUNCH_PAR
    return check_launch("ret_forward_parallel");
}

// ----------------------------------------------------------- recurrent form
//
// One block of 8 warps per (32 value columns, head, batch).  Lane l owns
// column j0 + l; warp w owns state rows w, w + 8, ...; the state stays in
// registers for the whole sequence.  Per token: S = gamma S + k v^T, then the
// column sums of q (.) S are reduced across the 8 warps.

constexpr int kRecMaxRows = 32;  // dk <= 256

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_recurrent_simt(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                        const Tin* __restrict__ v, HeadConsts hc, int N, int H,
                                                        int dk, int dv, Tout* __restrict__ out,
                                                        float* __restrict__ fstate, int xpos, long long pos0,
                                                        double log2base, int untaken_only) {
    const int h = blockIdx.y, b = blockIdx.z;
    // beside the tensor-core kernel: only the heads it leaves out
    if (untaken_only && hc.anchor[h] >= 0) return;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int j = blockIdx.x * 32 + lane;
    extern __shared__ double smd[];
    double* theta = smd;
    float* qs = reinterpret_cast<float*>(smd + (dk / 2 + 1));  // [2][dk]
    float* ks = qs + 2 * dk;                                     // [2][dk]
    float* red = ks + 2 * dk;                                    // [8][32]
    for (int p = threadIdx.x; p < dk / 2; p += blockDim.x) theta[p] = exp2(-2.0 * p / dk * log2base);
    const float g = (float)exp2(hc.log2g[h]);
    float S[kRecMaxRows];
#pragma unroll
    for (int i = 0; i < kRecMaxRows; i++) S[i] = 0.f;
    __syncthreads();
    for (int n = 0; n < N; n++) {
        float* qb = qs + (n & 1) * dk;
        float* kb = ks + (n & 1) * dk;
        load_rows_rotated(q, b, n, 1, N, H, h, dk, qb, dk, xpos != 0, pos0, theta);
        load_rows_rotated(k, b, n, 1, N, H, h, dk, kb, dk, xpos != 0, pos0, theta);
        const float vj = (j < dv) ? ld_as_float(v, (((size_t)b * N + n) * H + h) * dv + j) : 0.f;
        __syncthreads();
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kRecMaxRows; r++) {
            const int i = w + 8 * r;
            if (i < dk) {
                S[r] = fmaf(g, S[r], kb[i] * vj);
                acc = fmaf(qb[i], S[r], acc);
            }
        }
        red[w * 32 + lane] = acc;
        __syncthreads();
        if (w == 0 && j < dv) {
            float o = 0.f;
#pragma unroll
            for (int ww = 0; ww < 8; ww++) o += red[ww * 32 + lane];
            st_from_float(out, (((size_t)b * N + n) * H + h) * dv + j, o);
        }
    }
    if (fstate && j < dv) {
#pragma unroll
        for (int r = 0; r < kRecMaxRows; r++) {
            const int i = w + 8 * r;
            if (i < dk) fstate[(((size_t)b * H + h) * dk + i) * dv + j] = S[r];
        }
    }
}

ret_status launch_recurrent_simt(const RetArgs& a, cudaStream_t s, bool untaken_only) {
    if (a.dk > 8 * kRecMaxRows) return fail(RET_ERR_UNSUPPORTED, "ret_forward_recurrent: dk > 256");
    const size_t bytes = (size_t)(a.dk / 2 + 1) * sizeof(double) + ((size_t)4 * a.dk + 256) * sizeof(float);
    dim3 grid((a.dv + 31) / 32, a.H, a.B);
    const double lb = log2(a.theta_base);
#define RET_LAUNCH_REC(TI, TO)                                                                                \
    k_recurrent_simt<TI, TO><<<grid, 256, bytes, s>>>((const TI*)a.q, (const TI*)a.k, (const TI*)a.v, a.hc,  \
                                                      a.N, a.H, a.dk, a.dv, (TO*)a.out, a.final_state,       \
                                                      a.xpos, a.pos_offset, lb, untaken_only ? 1 : 0)
    if (a.in_dt == RET_F32 && a.out_dt == RET_F32) RET_LAUNCH_REC(float, float);
    else if (a.in_dt == RET_F32) RET_LAUNCH_REC(float, __nv_bfloat16);
    else if (a.out_dt == RET_F32) RET_LAUNCH_REC(__nv_bfloat16, float);
    else RET_LAUNCH_REC(__nv_bfloat16, __nv_bfloat16);
#undef RET_LAUNCH_REC
    return check_launch("ret_forward_recurrent");
}

}  // namespace ret
