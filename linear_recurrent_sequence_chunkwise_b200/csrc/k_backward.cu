// k_backward.cu -- gradients of chunkwise retention with respect to q, k, v,
// as tensor-core retention passes of the forward kernel.
//
// With q', k' the (rotated) vectors the recurrence multiplies ("Hybrid
// Architectures: RetNet and the Three Computation Paradigms", section 2.1;
// RetNet paper summary, Eq. 6) and dO the gradient of the output, the
// derivatives of o_n = sum_{m<=n} gamma^(n-m) (q'_n . k'_m) v_m are
//     dq'_n = sum_{m<=n} gamma^(n-m) (dO_n . v_m)   k'_m
//     dk'_m = sum_{n>=m} gamma^(n-m) (dO_n . v_m)   q'_n
//     dv_m  = sum_{n>=m} gamma^(n-m) (q'_n . k'_m)  dO_n
// Each is a retention with the same decay: dq' is the causal one with query
// dO, key v and value k'; dk' and dv are anti-causal, i.e. causal on the
// time-reversed sequence (query v, key dO, value q' and query k', key q',
// value dO).  dq' and dk' contract over d_v, which the tensor-core kernel
// takes in column slices of 128 or 256 (strided views of v and dO), each
// slice's result added into the fp32 gradient by the kernel's epilogue; the
// anti-causal passes store row n of their output at row N-1-n, i.e. back in
// time order.  With xPos, q' = R q and k' = R k, so dq = R^T dq' and
// dk = R^T dk' (the inverse rotation, section 6.8), applied in place at the
// end.  The dq and dv passes run on the caller's stream and the dk passes
// beside them on a second stream of the library's, joined back before the
// call returns: a pass of d_v slice width fills only B * H * dk / 64 SMs.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "kernels.h"

namespace ret {

namespace {

// Eight consecutive elements as fp32, through 16-byte accesses.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* x) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 f = __bfloat1622float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float* x) {
    const float4 u = reinterpret_cast<const float4*>(p)[0], w = reinterpret_cast<const float4*>(p)[1];
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    x[4] = w.x; x[5] = w.y; x[6] = w.z; x[7] = w.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* x) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float* x) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}

// Row transform, one warp per token t of batch b: reads row rs = (rev_src ?
// N-1-t : t) of `nsrc` source tensors (nsrc_stride elements apart) and sums
// them, turns each pair (2p, 2p+1) of every head by sign * (pos0 + t) *
// theta_p (sign 0: no rotation; -1: the inverse rotation), and writes the
// row to dst at (rev_dst ? N-1-t : t) and, if dst2 is set, to dst2 at N-1-t.
// With nsrc = 1 and rev_src == rev_dst, src and dst may be the same tensor.
// The sine and cosine of each (token, pair) are evaluated once for all
// heads; the loads of kHB heads are issued together.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_row_transform(const Tin* src, int nsrc, size_t nsrc_stride, Tout* dst,
                                                       Tout* __restrict__ dst2, int B, int N,
                                                       int H, int d, int rev_src, int rev_dst, float sign,
                                                       long long pos0, double log2base) {
    constexpr int kHB = 4;
    const int lane = threadIdx.x & 31;
    const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // b * N + t
    if (w >= (long long)B * N) return;
    const int b = (int)(w / N), t = (int)(w % N);
    const size_t rs = (size_t)b * N + (rev_src ? N - 1 - t : t);
    const size_t rd = (size_t)b * N + (rev_dst ? N - 1 - t : t);
    const size_t rd2 = (size_t)b * N + (N - 1 - t);
    for (int g = lane; g < d / 8; g += 32) {  // 8 elements = 4 pairs
        float cs[4], sn[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            cs[i] = 1.f;
            sn[i] = 0.f;
            if (sign != 0.f) {
                sincosf(rot_angle(pos0 + t, exp2(-2.0 * (4 * g + i) / d * log2base)), &sn[i], &cs[i]);
                sn[i] *= sign;
            }
        }
        for (int h0 = 0; h0 < H; h0 += kHB) {
            float x[kHB][8];
#pragma unroll
            for (int u = 0; u < kHB; u++)
#pragma unroll
                for (int e = 0; e < 8; e++) x[u][e] = 0.f;
            for (int j = 0; j < nsrc; j++) {
#pragma unroll
                for (int u = 0; u < kHB; u++) {
                    if (h0 + u >= H) break;
                    float y[8];
                    load8(src + j * nsrc_stride + (rs * H + h0 + u) * d + 8 * g, y);
#pragma unroll
                    for (int e = 0; e < 8; e++) x[u][e] += y[e];
                }
            }
#pragma unroll
            for (int u = 0; u < kHB; u++) {
                if (h0 + u >= H) break;
                float y[8];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    y[2 * i] = x[u][2 * i] * cs[i] - x[u][2 * i + 1] * sn[i];
                    y[2 * i + 1] = x[u][2 * i] * sn[i] + x[u][2 * i + 1] * cs[i];
                }
                store8(dst + (rd * H + h0 + u) * d + 8 * g, y);
                if (dst2) store8(dst2 + (rd2 * H + h0 + u) * d + 8 * g, y);
            }
        }
    }
}

template <typename Tin, typename Tout>
ret_status row_transform(const void* src, int nsrc, size_t nsrc_stride, void* dst, void* dst2, const BwdArgs& a, int d,
                         bool rev_src, bool rev_dst, float sign, cudaStream_t s) {
    const int blocks = (int)(((long long)a.B * a.N + 7) / 8);
    k_row_transform<Tin, Tout><<<blocks, 256, 0, s>>>(reinterpret_cast<const Tin*>(src), nsrc, nsrc_stride,
                                                      reinterpret_cast<Tout*>(dst), reinterpret_cast<Tout*>(dst2),
                                                      a.B, a.N, a.H, d, rev_src, rev_dst, a.xpos ? sign : 0.f,
                                                      a.pos_offset, log2(a.theta_base));
    return check_launch("backward: row transform");
}

// The contraction slice of d_v taken per tensor-core pass.
int dv_slice(int dv) { return dv % 256 == 0 ? 256 : 128; }

struct BwdLayout {
    size_t kr, kr_rev, qr_rev, v_rev, do_rev, inner, inner2, total;
};

BwdLayout bwd_layout(const BwdArgs& a) {
    const size_t tok = (size_t)a.B * a.N * a.H, qk = tok * a.dk * 2, vv = tok * a.dv * 2;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    BwdLayout L;
    size_t o = 0;
    L.kr = o; o += al(qk);
    L.kr_rev = o; o += al(qk);
    L.qr_rev = o; o += al(qk);
    L.v_rev = o; o += al(vv);
    L.do_rev = o; o += al(vv);
    const size_t inner = al(std::max(qk, tok * dv_slice(a.dv) * 2));  // k' of one pass
    L.inner = o; o += inner;
    L.inner2 = o; o += inner;  // the second stream's passes
    L.total = o;
    return L;
}

// One causal retention pass of the workspace path (prep, then the
// tensor-core kernel) with query/key rows q_ld / k_ld elements apart; its
// fp32 output is stored (or added, `accumulate`) at row n, or at row N-1-n
// (`out_rev`).
ret_status pass(const BwdArgs& b, const void* q, int q_ld, const void* k, int k_ld, int dk, const void* v, int dv,
                float* out, bool accumulate, bool out_rev, void* inner, cudaStream_t s) {
    RetArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.out = out;
    a.B = b.B; a.N = b.N; a.H = b.H; a.dk = dk; a.dv = dv; a.chunk = b.chunk;
    a.in_dt = RET_BF16; a.out_dt = RET_F32;
    a.xpos = 0; a.theta_base = 10000.0;
    a.hc = b.hc;
    a.q_ld = q_ld; a.k_ld = k_ld; a.accumulate = accumulate ? 1 : 0; a.out_rev = out_rev ? 1 : 0;
    if (!chunkwise_ws_supported(a)) return fail(RET_ERR_UNSUPPORTED, "backward: pass shape outside the tensor-core path");
    ret_status st = launch_chunkwise_prep(a, inner, s);
    if (st != RET_OK) return st;
    return launch_chunkwise_prepared(a, inner, s);
}

// A second stream per device for the dk passes, which run beside the dq
// passes (each pass fills only B * H * dk / 64 SMs).
ret_status side_stream(cudaStream_t* out) {
    constexpr int kMaxDev = 64;
    static cudaStream_t streams[kMaxDev];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return fail(RET_ERR_CUDA, "backward: no current device");
    std::lock_guard<std::mutex> lock(mu);
    if (!streams[dev] && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess) {
        streams[dev] = nullptr;
        return check_launch("backward: creating the second stream");
    }
    *out = streams[dev];
    return RET_OK;
}

// `to` waits for everything enqueued on `from` so far.
ret_status join(cudaStream_t from, cudaStream_t to) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return check_launch("backward: event");
    const bool ok = cudaEventRecord(e, from) == cudaSuccess && cudaStreamWaitEvent(to, e, 0) == cudaSuccess;
    cudaEventDestroy(e);  // released once it has completed
    return ok ? RET_OK : check_launch("backward: stream join");
}

}  // namespace

bool backward_supported(const BwdArgs& a) {
    if (a.chunk != 128 || !(a.dk == 128 || a.dk == 256) || a.dv % 128 != 0) return false;
    for (int h = 0; h < a.H; h++)
        if (!(a.hc.log2g[h] * a.chunk >= -60.0)) return false;
    return true;
}

size_t backward_ws_bytes(const BwdArgs& a) { return bwd_layout(a).total; }

ret_status launch_backward(const BwdArgs& a, cudaStream_t s) {
    const BwdLayout L = bwd_layout(a);
    uint8_t* ws = reinterpret_cast<uint8_t*>(a.workspace);
    auto at = [&](size_t off) { return reinterpret_cast<void*>(ws + off); };
    using bf = __nv_bfloat16;
    ret_status st;
    cudaStream_t s2;
    if ((st = side_stream(&s2)) != RET_OK || (st = join(s, s2)) != RET_OK) return st;

    // Caller's stream: k' = R k in both time orders, then the dq passes.
    // Second stream: q' = R q, v and dO reversed, then the dk passes.
    if ((st = row_transform<bf, bf>(a.k, 1, 0, at(L.kr), at(L.kr_rev), a, a.dk, false, false, 1.f, s)) != RET_OK ||
        (st = row_transform<bf, bf>(a.q, 1, 0, at(L.qr_rev), nullptr, a, a.dk, false, true, 1.f, s2)) != RET_OK ||
        (st = row_transform<bf, bf>(a.dout, 1, 0, at(L.do_rev), nullptr, a, a.dv, false, true, 0.f, s2)) != RET_OK)
        return st;
    cudaEvent_t reversed;  // q' and dO reversed: what the dv pass takes from the second stream
    if (cudaEventCreateWithFlags(&reversed, cudaEventDisableTiming) != cudaSuccess)
        return check_launch("backward: event");
    const bool rec = cudaEventRecord(reversed, s2) == cudaSuccess;
    if (!rec || (st = row_transform<bf, bf>(a.v, 1, 0, at(L.v_rev), nullptr, a, a.dv, false, true, 0.f, s2)) != RET_OK) {
        cudaEventDestroy(reversed);
        return rec ? st : check_launch("backward: event record");
    }

    const int S = dv_slice(a.dv), nsl = a.dv / S;
    const bf* dout = reinterpret_cast<const bf*>(a.dout);
    const bf* v = reinterpret_cast<const bf*>(a.v);
    const bf* v_rev = reinterpret_cast<const bf*>(at(L.v_rev));
    const bf* do_rev = reinterpret_cast<const bf*>(at(L.do_rev));
    for (int i = 0; i < nsl && st == RET_OK; i++) {
        const int s0 = i * S;
        // dq' = causal retention (query dO, key v, value k'), d_v slice [s0, s0 + S)
        st = pass(a, dout + s0, a.dv, v + s0, a.dv, S, at(L.kr), a.dk, a.dq, i > 0, false, at(L.inner), s);
        // dk' = causal retention (query v, key dO, value q') on the reversed sequence, stored back in time order
        if (st == RET_OK)
            st = pass(a, v_rev + s0, a.dv, do_rev + s0, a.dv, S, at(L.qr_rev), a.dk, a.dkk, i > 0, true, at(L.inner2),
                      s2);
    }
    // dv = causal retention (query k', key q', value dO) on the reversed sequence, stored back in time order
    if (st == RET_OK && cudaStreamWaitEvent(s, reversed, 0) != cudaSuccess) st = check_launch("backward: stream wait");
    cudaEventDestroy(reversed);  // released once it has completed
    if (st == RET_OK)
        st = pass(a, at(L.kr_rev), a.dk, at(L.qr_rev), a.dk, a.dk, at(L.do_rev), a.dv, a.dvv, false, true, at(L.inner),
                  s);
    if (st != RET_OK) return st;
    if (a.xpos) {  // dq = R^T dq', dk = R^T dk', in place
        if ((st = row_transform<float, float>(a.dkk, 1, 0, a.dkk, nullptr, a, a.dk, false, false, -1.f, s2)) != RET_OK ||
            (st = row_transform<float, float>(a.dq, 1, 0, a.dq, nullptr, a, a.dk, false, false, -1.f, s)) != RET_OK)
            return st;
    }
    return join(s2, s);  // the caller's stream covers the second stream's work
}

}  // namespace ret
