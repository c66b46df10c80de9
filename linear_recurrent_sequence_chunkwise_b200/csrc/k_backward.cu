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
// takes in column slices of 128 or 256 (strided views of v and dO), adding
// the slices in fp32.  With xPos, q' = R q and k' = R k, so dq = R^T dq' and
// dk = R^T dk' (the inverse rotation, section 6.8).
#include <algorithm>
#include <cstring>

#include "kernels.h"

namespace ret {

namespace {

// dst[b][N-1-n][:] = src[b][n][:] for rows of row_vec 16-byte vectors.
__global__ void k_reverse_rows(const uint4* __restrict__ src, uint4* __restrict__ dst, long long N, size_t row_vec,
                               size_t total_vec) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total_vec; i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / row_vec, c = i % row_vec;  // row = b * N + n
        const size_t b = row / (size_t)N, n = row % (size_t)N;
        dst[(b * (size_t)N + ((size_t)N - 1 - n)) * row_vec + c] = __ldg(src + i);
    }
}

ret_status reverse_rows(const void* src, void* dst, int B, int N, size_t row_bytes, cudaStream_t s) {
    const size_t row_vec = row_bytes / 16, total = (size_t)B * N * row_vec;
    const int threads = 256;
    const int blocks = (int)std::min<size_t>((total + threads - 1) / threads, 148 * 32);
    k_reverse_rows<<<blocks, threads, 0, s>>>(reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), N,
                                              row_vec, total);
    return check_launch("backward: reverse rows");
}

// The contraction slice of d_v taken per tensor-core pass.
int dv_slice(int dv) { return dv % 256 == 0 ? 256 : 128; }

struct BwdLayout {
    size_t qr, kr, qr_rev, kr_rev, v_rev, do_rev, inner, dk_rev, dv_rev, total;
};

BwdLayout bwd_layout(const BwdArgs& a) {
    const size_t qk = (size_t)a.B * a.N * a.H * a.dk * 2, vv = (size_t)a.B * a.N * a.H * a.dv * 2;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    BwdLayout L;
    size_t o = 0;
    L.qr = o; o += al(qk);
    L.kr = o; o += al(qk);
    L.qr_rev = o; o += al(qk);
    L.kr_rev = o; o += al(qk);
    L.v_rev = o; o += al(vv);
    L.do_rev = o; o += al(vv);
    L.inner = o; o += al(std::max(qk, (size_t)a.B * a.N * a.H * dv_slice(a.dv) * 2));  // k' of one pass
    L.dk_rev = o; o += al(2 * qk);  // fp32
    L.dv_rev = o; o += al(2 * vv);  // fp32
    L.total = o;
    return L;
}

// One causal retention pass of the workspace path (prep, then the
// tensor-core kernel) with query/key rows q_ld / k_ld elements apart.
ret_status pass(const BwdArgs& b, const void* q, int q_ld, const void* k, int k_ld, int dk, const void* v, int dv,
                float* out, bool accumulate, void* inner, cudaStream_t s) {
    RetArgs a;
    memset(&a, 0, sizeof(a));
    a.q = q; a.k = k; a.v = v; a.out = out;
    a.B = b.B; a.N = b.N; a.H = b.H; a.dk = dk; a.dv = dv; a.chunk = b.chunk;
    a.in_dt = RET_BF16; a.out_dt = RET_F32;
    a.xpos = 0; a.theta_base = 10000.0;
    a.hc = b.hc;
    a.q_ld = q_ld; a.k_ld = k_ld; a.accumulate = accumulate ? 1 : 0;
    if (!chunkwise_ws_supported(a)) return fail(RET_ERR_UNSUPPORTED, "backward: pass shape outside the tensor-core path");
    ret_status st = launch_chunkwise_prep(a, inner, s);
    if (st != RET_OK) return st;
    return launch_chunkwise_prepared(a, inner, s);
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
    const size_t qk = (size_t)a.B * a.N * a.H * a.dk * 2;
    const size_t qrow = (size_t)a.H * a.dk, vrow = (size_t)a.H * a.dv;  // elements per (b, n) row
    ret_status st;

    // q' and k': copies, rotated in place with xPos.
    if (cudaMemcpyAsync(at(L.qr), a.q, qk, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(at(L.kr), a.k, qk, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return check_launch("backward: copies of q and k");
    if (a.xpos) {
        if ((st = launch_xpos_rotate(at(L.qr), RET_BF16, a.B, a.N, a.H, a.dk, a.pos_offset, a.theta_base, s)) != RET_OK ||
            (st = launch_xpos_rotate(at(L.kr), RET_BF16, a.B, a.N, a.H, a.dk, a.pos_offset, a.theta_base, s)) != RET_OK)
            return st;
    }
    // Time-reversed sequences for the two anti-causal sums.
    if ((st = reverse_rows(at(L.qr), at(L.qr_rev), a.B, a.N, qrow * 2, s)) != RET_OK ||
        (st = reverse_rows(at(L.kr), at(L.kr_rev), a.B, a.N, qrow * 2, s)) != RET_OK ||
        (st = reverse_rows(a.v, at(L.v_rev), a.B, a.N, vrow * 2, s)) != RET_OK ||
        (st = reverse_rows(a.dout, at(L.do_rev), a.B, a.N, vrow * 2, s)) != RET_OK)
        return st;

    const int S = dv_slice(a.dv);
    const __nv_bfloat16* dout = reinterpret_cast<const __nv_bfloat16*>(a.dout);
    const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(a.v);
    const __nv_bfloat16* v_rev = reinterpret_cast<const __nv_bfloat16*>(at(L.v_rev));
    const __nv_bfloat16* do_rev = reinterpret_cast<const __nv_bfloat16*>(at(L.do_rev));
    for (int s0 = 0; s0 < a.dv; s0 += S) {
        // dq' = causal retention (query dO, key v, value k'), d_v slice [s0, s0 + S)
        if ((st = pass(a, dout + s0, a.dv, v + s0, a.dv, S, at(L.kr), a.dk, a.dq, s0 > 0, at(L.inner), s)) != RET_OK)
            return st;
        // reversed dk' = causal retention (query v, key dO, value q') on the reversed sequence
        if ((st = pass(a, v_rev + s0, a.dv, do_rev + s0, a.dv, S, at(L.qr_rev), a.dk,
                       reinterpret_cast<float*>(at(L.dk_rev)), s0 > 0, at(L.inner), s)) != RET_OK)
            return st;
    }
    // reversed dv = causal retention (query k', key q', value dO) on the reversed sequence
    if ((st = pass(a, at(L.kr_rev), a.dk, at(L.qr_rev), a.dk, a.dk, at(L.do_rev), a.dv,
                   reinterpret_cast<float*>(at(L.dv_rev)), false, at(L.inner), s)) != RET_OK)
        return st;
    if ((st = reverse_rows(at(L.dk_rev), a.dkk, a.B, a.N, qrow * 4, s)) != RET_OK ||
        (st = reverse_rows(at(L.dv_rev), a.dvv, a.B, a.N, vrow * 4, s)) != RET_OK)
        return st;
    if (a.xpos) {
        if ((st = launch_xpos_rotate(a.dq, RET_F32, a.B, a.N, a.H, a.dk, a.pos_offset, a.theta_base, s, true)) !=
                RET_OK ||
            (st = launch_xpos_rotate(a.dkk, RET_F32, a.B, a.N, a.H, a.dk, a.pos_offset, a.theta_base, s, true)) !=
                RET_OK)
            return st;
    }
    return RET_OK;
}

}  // namespace ret
