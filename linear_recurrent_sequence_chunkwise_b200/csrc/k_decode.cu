// k_decode.cu -- recurrent decode step ("Hybrid Architectures: RetNet and the
// Three Computation Paradigms", sections 2.1 and 5.2; RetNet paper summary,
// inference protocol): S <- gamma S + k v^T, then o = q^T S.
//
// HBM-bound: each step reads and writes the fp32 state once (0.5 FLOP/byte).
// A block of 8 warps covers 128 value columns of one (batch, head): lane l
// owns four consecutive columns (one 16-byte vector), warp w a contiguous
// band of dk/8 state rows, so every warp-wide access is a coalesced 512-byte
// row segment.  Each thread keeps a batch of 16 row vectors in flight, then
// the per-warp partial sums of q (.) S are reduced across the 8 warps in
// shared memory.
#include "kernels.h"

namespace ret {

constexpr int kDecCols = 128;   // columns per block (32 lanes x 4)
constexpr int kDecWarps = 8;
constexpr int kDecBatch = 16;   // row vectors in flight per thread

__device__ __forceinline__ float4 ld_stream(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4* p, float4 x) { __stcs(p, x); }

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_decode_step(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                     const Tin* __restrict__ v, HeadConsts hc, int H, int dk,
                                                     int dv, float* __restrict__ state, Tout* __restrict__ out) {
    extern __shared__ float smf[];
    float* qs = smf;            // [dk]
    float* ks = smf + dk;       // [dk]
    float4* red = reinterpret_cast<float4*>(smf + ((2 * dk + 3) & ~3));  // [8][32], 16-byte aligned
    const int bh = blockIdx.y, h = bh % H;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int j = blockIdx.x * kDecCols + lane * 4;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        qs[i] = ld_as_float(q, (size_t)bh * dk + i);
        ks[i] = ld_as_float(k, (size_t)bh * dk + i);
    }
    const float g = (float)exp2(hc.log2g[h]);
    __syncthreads();

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < dv) {
        const size_t vb = (size_t)bh * dv + j;
        const float v0 = ld_as_float(v, vb), v1 = ld_as_float(v, vb + 1);
        const float v2 = ld_as_float(v, vb + 2), v3 = ld_as_float(v, vb + 3);
        const int rows = (dk + kDecWarps - 1) / kDecWarps;
        const int i0 = w * rows, i1 = min(dk, i0 + rows);
        float4* S = reinterpret_cast<float4*>(state + (size_t)bh * dk * dv + j);
        const int ld4 = dv / 4;
        for (int ib = i0; ib < i1; ib += kDecBatch) {
            float4 s[kDecBatch];
#pragma unroll
            for (int t = 0; t < kDecBatch; t++)
                if (ib + t < i1) s[t] = ld_stream(S + (size_t)(ib + t) * ld4);
#pragma unroll
            for (int t = 0; t < kDecBatch; t++) {
                const int i = ib + t;
                if (i < i1) {
                    const float ki = ks[i], qi = qs[i];
                    float4 x = s[t];
                    x.x = fmaf(g, x.x, ki * v0);
                    x.y = fmaf(g, x.y, ki * v1);
                    x.z = fmaf(g, x.z, ki * v2);
                    x.w = fmaf(g, x.w, ki * v3);
                    st_stream(S + (size_t)i * ld4, x);
                    acc.x = fmaf(qi, x.x, acc.x);
                    acc.y = fmaf(qi, x.y, acc.y);
                    acc.z = fmaf(qi, x.z, acc.z);
                    acc.w = fmaf(qi, x.w, acc.w);
                }
            }
        }
    }
    red[w * 32 + lane] = acc;
    __syncthreads();
    if (w == 0 && j < dv) {
        float4 o = red[lane];
#pragma unroll
        for (int ww = 1; ww < kDecWarps; ww++) {
            const float4 r = red[ww * 32 + lane];
            o.x += r.x; o.y += r.y; o.z += r.z; o.w += r.w;
        }
        const size_t ob = (size_t)bh * dv + j;
        st_from_float(out, ob, o.x);
        st_from_float(out, ob + 1, o.y);
        st_from_float(out, ob + 2, o.z);
        st_from_float(out, ob + 3, o.w);
    }
}

ret_status launch_decode(const void* q, const void* k, const void* v, const HeadConsts& hc, float* state,
                         void* out, int B, int H, int dk, int dv, ret_dtype in_dt, ret_dtype out_dt,
                         cudaStream_t s) {
    dim3 grid((dv + kDecCols - 1) / kDecCols, B * H);
    const size_t smem = (size_t)((2 * dk + 3) & ~3) * sizeof(float) + kDecWarps * 32 * sizeof(float4);
    if (smem > 48 * 1024) return fail(RET_ERR_UNSUPPORTED, "ret_decode_step: dk too large");
#define RET_LAUNCH_DEC(TI, TO)                                                                               \
    k_decode_step<TI, TO><<<grid, 256, smem, s>>>((const TI*)q, (const TI*)k, (const TI*)v, hc, H, dk, dv, \
                                                  state, (TO*)out)
    if (in_dt == RET_F32 && out_dt == RET_F32) RET_LAUNCH_DEC(float, float);
    else if (in_dt == RET_F32) RET_LAUNCH_DEC(float, __nv_bfloat16);
    else if (out_dt == RET_F32) RET_LAUNCH_DEC(__nv_bfloat16, float);
    else RET_LAUNCH_DEC(__nv_bfloat16, __nv_bfloat16);
#undef RET_LAUNCH_DEC
    return check_launch("ret_decode_step");
}

}  // namespace ret
