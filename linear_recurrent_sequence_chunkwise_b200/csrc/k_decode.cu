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

// With xpos, q and k of sequence b are first turned by the xPos rotation at
// its position (section 6.8).  With flags (the score normalizations 2 and 3
// of section 8.5), the output is multiplied by f = c / max(|c q.z|, 1),
// c = 1 / sqrt(sum_{i<=pos} gamma^i), where z is the decayed key sum already
// updated for this token.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_decode_step(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                     const Tin* __restrict__ v, HeadConsts hc, int H, int dk,
                                                     int dv, float* __restrict__ state, Tout* __restrict__ out,
                                                     DecodeOpts o) {
    const float* __restrict__ z = o.z;
    const int flags = o.flags;
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
    const long long pos = o.positions ? o.positions[bh / H] : o.pos;
    if (o.xpos) {
        __syncthreads();
        for (int p = threadIdx.x; p < dk / 2; p += blockDim.x) {
            float sn, cs;
            sincosf(rot_angle(pos, exp2(-2.0 * p / dk * o.log2base)), &sn, &cs);
            const float q0 = qs[2 * p], q1 = qs[2 * p + 1], k0 = ks[2 * p], k1 = ks[2 * p + 1];
            qs[2 * p] = q0 * cs - q1 * sn;
            qs[2 * p + 1] = q0 * sn + q1 * cs;
            ks[2 * p] = k0 * cs - k1 * sn;
            ks[2 * p + 1] = k0 * sn + k1 * cs;
        }
    }
    __syncthreads();
    float fscale = 1.f;
    if (flags) {
        __shared__ float s_part[kDecWarps], s_f;
        float part = 0.f;
        if (flags & kNormScore)
            for (int i = threadIdx.x; i < dk; i += blockDim.x) part = fmaf(qs[i], z[(size_t)bh * dk + i], part);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) s_part[w] = part;
        __syncthreads();
        if (threadIdx.x == 0) {
            float sn = 0.f;
            for (int ww = 0; ww < kDecWarps; ww++) sn += s_part[ww];
            const double lg = hc.log2g[h];
            double f = 1.0;
            if (flags & kNormDecay) {
                const double ln_g = lg * 0.69314718055994530942, cnt = (double)(pos + 1);
                f = 1.0 / sqrt(lg == 0.0 ? cnt : expm1(cnt * ln_g) / expm1(ln_g));
            }
            if (flags & kNormScore) f /= fmax(fabs(f * (double)sn), 1.0);
            s_f = (float)f;
        }
        __syncthreads();
        fscale = s_f;
    }

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
        o.x *= fscale; o.y *= fscale; o.z *= fscale; o.w *= fscale;
        const size_t ob = (size_t)bh * dv + j;
        st_from_float(out, ob, o.x);
        st_from_float(out, ob + 1, o.y);
        st_from_float(out, ob + 2, o.z);
        st_from_float(out, ob + 3, o.w);
    }
}

// z <- gamma z + k (k rotated at its sequence's position with xpos), one
// thread per pair of elements of z [B, H, dk].
template <typename Tin>
__global__ void k_keysum_update(float* __restrict__ z, const Tin* __restrict__ k, HeadConsts hc, int H, int dk,
                                long long total_pairs, DecodeOpts o) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total_pairs) return;
    const int half = (dk + 1) / 2;  // an odd dk (no rotation then) leaves a last single element
    const int p = (int)(i % half);
    const long long bh = i / half;
    const int h = (int)(bh % H);
    const size_t e = (size_t)bh * dk + 2 * p;
    const bool pair = 2 * p + 1 < dk;
    float k0 = ld_as_float(k, e), k1 = pair ? ld_as_float(k, e + 1) : 0.f;
    if (o.xpos) {
        const long long pos = o.positions ? o.positions[bh / H] : o.pos;
        float sn, cs;
        sincosf(rot_angle(pos, exp2(-2.0 * p / dk * o.log2base)), &sn, &cs);
        const float r0 = k0 * cs - k1 * sn, r1 = k0 * sn + k1 * cs;
        k0 = r0;
        k1 = r1;
    }
    const float g = (float)exp2(hc.log2g[h]);
    z[e] = fmaf(g, z[e], k0);
    if (pair) z[e + 1] = fmaf(g, z[e + 1], k1);
}

static ret_status decode_launch(const void* q, const void* k, const void* v, const HeadConsts& hc, float* state,
                                void* out, int B, int H, int dk, int dv, ret_dtype in_dt, ret_dtype out_dt,
                                const DecodeOpts& o, cudaStream_t s);

ret_status launch_decode(const void* q, const void* k, const void* v, const HeadConsts& hc, float* state,
                         void* out, int B, int H, int dk, int dv, ret_dtype in_dt, ret_dtype out_dt,
                         cudaStream_t s) {
    DecodeOpts o{};
    return decode_launch(q, k, v, hc, state, out, B, H, dk, dv, in_dt, out_dt, o, s);
}

ret_status launch_decode_ex(const void* q, const void* k, const void* v, const HeadConsts& hc, float* state,
                            void* out, int B, int H, int dk, int dv, ret_dtype in_dt, ret_dtype out_dt,
                            const DecodeOpts& o, cudaStream_t s) {
    if (o.flags & kNormScore) {
        const long long total = (long long)B * H * ((dk + 1) / 2);
        const int blocks = (int)((total + 255) / 256);
        if (in_dt == RET_F32)
            k_keysum_update<float><<<blocks, 256, 0, s>>>(o.z, (const float*)k, hc, H, dk, total, o);
        else
            k_keysum_update<__nv_bfloat16><<<blocks, 256, 0, s>>>(o.z, (const __nv_bfloat16*)k, hc, H, dk, total, o);
        ret_status st = check_launch("decode: key sum");
        if (st != RET_OK) return st;
    }
    return decode_launch(q, k, v, hc, state, out, B, H, dk, dv, in_dt, out_dt, o, s);
}

static ret_status decode_launch(const void* q, const void* k, const void* v, const HeadConsts& hc, float* state,
                                void* out, int B, int H, int dk, int dv, ret_dtype in_dt, ret_dtype out_dt,
                                const DecodeOpts& o, cudaStream_t s) {
    dim3 grid((dv + kDecCols - 1) / kDecCols, B * H);
    const size_t smem = (size_t)((2 * dk + 3) & ~3) * sizeof(float) + kDecWarps * 32 * sizeof(float4);
    if (smem > 48 * 1024) return fail(RET_ERR_UNSUPPORTED, "ret_decode_step: dk too large");
#define RET_LAUNCH_DEC(TI, TO)                                                                               \
    k_decode_step<TI, TO><<<grid, 256, smem, s>>>((const TI*)q, (const TI*)k, (const TI*)v, hc, H, dk, dv, \
                                                  state, (TO*)out, o)
    if (in_dt == RET_F32 && out_dt == RET_F32) RET_LAUNCH_DEC(float, float);
    else if (in_dt == RET_F32) RET_LAUNCH_DEC(float, __nv_bfloat16);
    else if (out_dt == RET_F32) RET_LAUNCH_DEC(__nv_bfloat16, float);
    else RET_LAUNCH_DEC(__nv_bfloat16, __nv_bfloat16);
#undef RET_LAUNCH_DEC
    return check_launch("ret_decode_step");
}

}  // namespace ret
