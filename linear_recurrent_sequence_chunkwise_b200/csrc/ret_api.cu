// ret_api.cu -- the C ABI: argument validation, per-head constants and
// dispatch to the kernels.  Nothing here allocates device memory, apart from
// ret_forward_chunkwise's stream-ordered scratch from the library's pool
// (see k_chunk_ws.cu).
#include <cstring>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include "gemm.h"
#include "kernels.h"

namespace ret {

static thread_local char t_err[512] = "";

ret_status fail(ret_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof(t_err), fmt, ap);
    va_end(ap);
    return st;
}

ret_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return RET_OK;
}

bool make_head_consts(const double* gammas, int H, HeadConsts* hc) {
    if (H < 1 || H > kMaxHeads) return false;
    for (int h = 0; h < H; h++) hc->log2g[h] = log2(gammas[h]);  // -inf for gamma = 0
    for (int h = H; h < kMaxHeads; h++) hc->log2g[h] = 0.0;
    for (int h = 0; h < kMaxHeads; h++) hc->anchor[h] = decay_anchor(hc->log2g[h]);
    return true;
}

static bool is_dtype(ret_dtype d) { return d == RET_F32 || d == RET_BF16; }
static size_t esize(ret_dtype d) { return d == RET_F32 ? 4 : 2; }

static bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const char* pa = (const char*)a;
    const char* pb = (const char*)b;
    return pa < pb + nb && pb < pa + na;
}

static ret_status check_gammas(const double* gammas, int H, const char* who) {
    if (!gammas) return fail(RET_ERR_INVALID_ARG, "%s: gammas is NULL", who);
    if (H < 1 || H > kMaxHeads) return fail(RET_ERR_INVALID_ARG, "%s: H=%d outside [1, %d]", who, H, kMaxHeads);
    for (int h = 0; h < H; h++)
        if (!(gammas[h] >= 0.0 && gammas[h] <= 1.0))
            return fail(RET_ERR_INVALID_ARG, "%s: gammas[%d]=%g outside [0, 1]", who, h, gammas[h]);
    return RET_OK;
}

// Shared validation of the sequence-level entry points.
static ret_status make_args(RetArgs* a, const char* who, const void* q, const void* k, const void* v,
                            const double* gammas, int B, int N, int H, int dk, int dv, int chunk, void* out,
                            float* final_state, ret_dtype in_dt, ret_dtype out_dt, int xpos, int64_t pos_offset,
                            double theta_base) {
    if (!q || !k || !v || !out) return fail(RET_ERR_INVALID_ARG, "%s: NULL q, k, v or out", who);
    if (B < 1 || N < 1 || H < 1 || dk < 1 || dv < 1 || chunk < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1 (B=%d N=%d H=%d dk=%d dv=%d chunk=%d)", who, B,
                    N, H, dk, dv, chunk);
    if (!is_dtype(in_dt) || !is_dtype(out_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (xpos && (dk % 2 != 0)) return fail(RET_ERR_INVALID_ARG, "%s: xpos needs an even dk (got %d)", who, dk);
    if (xpos && !(theta_base > 0.0 && isfinite(theta_base)))
        return fail(RET_ERR_INVALID_ARG, "%s: theta_base must be finite and > 0", who);
    const size_t ntok = (size_t)B * N * H;
    if (ntok * (size_t)(dk > dv ? dk : dv) > ((size_t)1 << 40))
        return fail(RET_ERR_INVALID_ARG, "%s: problem too large", who);
    for (const void* p : {q, k, v, (const void*)out})
        if (!aligned(p, 16)) return fail(RET_ERR_INVALID_ARG, "%s: device pointers must be 16-byte aligned", who);
    if (final_state && !aligned(final_state, 16))
        return fail(RET_ERR_INVALID_ARG, "%s: final_state must be 16-byte aligned", who);
    const size_t bq = ntok * dk * esize(in_dt), bv = ntok * dv * esize(in_dt), bo = ntok * dv * esize(out_dt);
    if (overlaps(out, bo, q, bq) || overlaps(out, bo, k, bq) || overlaps(out, bo, v, bv))
        return fail(RET_ERR_INVALID_ARG, "%s: out overlaps q, k or v", who);
    if (final_state) {
        const size_t bs = (size_t)B * H * dk * dv * 4;
        if (overlaps(final_state, bs, out, bo) || overlaps(final_state, bs, q, bq) ||
            overlaps(final_state, bs, k, bq) || overlaps(final_state, bs, v, bv))
            return fail(RET_ERR_INVALID_ARG, "%s: final_state overlaps another buffer", who);
    }
    a->q = q; a->k = k; a->v = v; a->out = out; a->final_state = final_state; a->initial_state = nullptr;
    a->q_ld = 0; a->k_ld = 0; a->accumulate = 0; a->out_rev = 0; a->rowscale = nullptr; a->dk_real = 0;
    a->B = B; a->N = N; a->H = H; a->dk = dk; a->dv = dv; a->chunk = chunk;
    a->in_dt = in_dt; a->out_dt = out_dt;
    a->xpos = xpos ? 1 : 0; a->pos_offset = pos_offset; a->theta_base = xpos ? theta_base : 10000.0;
    make_head_consts(gammas, H, &a->hc);
    for (int h = 0; h < kMaxHeads; h++) a->gamma[h] = h < H ? gammas[h] : 0.0;
    return RET_OK;
}

}  // namespace ret

using namespace ret;

// The workspace path's kernel takes d_k = 128 or 256.  A d_k of 64 runs on it
// zero-padded to 128: the padded components add nothing to q . k and leave
// the padded state rows at zero.  Its kernel blocks the sequence by 128
// tokens, so a chunk of 64 is computed in blocks of 128 (the chunkwise form
// gives the recurrence's result for any block length).
static void pad_small_dk(RetArgs* a) {
    if (a->in_dt == RET_BF16 && a->dk == 64 && (a->chunk == 64 || a->chunk == 128)) {
        a->dk_real = 64;
        a->dk = 128;
        a->chunk = 128;
    }
}

extern "C" {

const char* ret_last_error_string(void) { return t_err; }

ret_status ret_xpos_rotate(void* x, ret_dtype dt, int B, int N, int H, int d, int64_t pos_offset, double theta_base,
                           cudaStream_t stream) {
    t_err[0] = 0;
    if (!x) return fail(RET_ERR_INVALID_ARG, "ret_xpos_rotate: x is NULL");
    if (!is_dtype(dt)) return fail(RET_ERR_INVALID_ARG, "ret_xpos_rotate: unknown dtype");
    if (B < 1 || N < 1 || H < 1 || d < 2 || d % 2)
        return fail(RET_ERR_INVALID_ARG, "ret_xpos_rotate: sizes must be >= 1 and d even >= 2");
    if (!(theta_base > 0.0 && isfinite(theta_base)))
        return fail(RET_ERR_INVALID_ARG, "ret_xpos_rotate: theta_base must be finite and > 0");
    if (!aligned(x, 4)) return fail(RET_ERR_INVALID_ARG, "ret_xpos_rotate: x must be 4-byte aligned");
    return launch_xpos_rotate(x, dt, B, N, H, d, pos_offset, theta_base, stream);
}

ret_status ret_forward_chunkwise(const void* q, const void* k, const void* v, const double* gammas, int B, int N,
                                 int H, int dk, int dv, int chunk, void* out, float* final_state,
                                 cudaStream_t stream, ret_dtype in_dt, ret_dtype out_dt, int xpos,
                                 int64_t pos_offset, double theta_base) {
    t_err[0] = 0;
    RetArgs a;
    ret_status st = make_args(&a, "ret_forward_chunkwise", q, k, v, gammas, B, N, H, dk, dv, chunk, out,
                              final_state, in_dt, out_dt, xpos, pos_offset, theta_base);
    if (st != RET_OK) return st;
    {
        // the tensor-core path, scores form (d_k = 64 padded to 128);
        // heads too fast for it (gamma^64 < 2^-100), if any, token by token
        RetArgs f = a;
        pad_small_dk(&f);
        const int left = chunkwise_heads_below(f, 0);
        if (chunkwise_ws_shape_ok(f) && left < H) {
            st = launch_chunkwise_scores_pooled(f, stream);
            if (st != RET_OK || left == 0) return st;
            return launch_recurrent_simt(a, stream, true);
        }
    }
    st = launch_chunkwise_simt(a, stream);
    if (st != RET_ERR_UNSUPPORTED) return st;
    // Same function, token by token: the shape fits neither chunkwise kernel.
    t_err[0] = 0;
    return launch_recurrent_simt(a, stream);
}

// The caller's d_k (before padding).
static int dk_of(const RetArgs& a) { return a.dk_real ? a.dk_real : a.dk; }

size_t ret_chunkwise_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk, ret_dtype in_dt, int xpos) {
    if (B < 1 || N < 1 || H < 1 || H > kMaxHeads || dk < 1 || dv < 1 || chunk < 1) return 0;
    RetArgs a{};
    a.B = B; a.N = N; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.in_dt = in_dt; a.xpos = xpos ? 1 : 0;
    for (int h = 0; h < kMaxHeads; h++) a.hc.log2g[h] = 0.0, a.hc.anchor[h] = kChunkAnchorFull;  // shape check only
    pad_small_dk(&a);
    return chunkwise_ws_supported(a) ? chunkwise_scores_bytes(a) : 0;
}

size_t ret_chunkwise_prepare_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk, ret_dtype in_dt,
                                             int xpos) {
    if (B < 1 || N < 1 || H < 1 || H > kMaxHeads || dk < 1 || dv < 1 || chunk < 1) return 0;
    RetArgs a{};
    a.B = B; a.N = N; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.in_dt = in_dt; a.xpos = xpos ? 1 : 0;
    for (int h = 0; h < kMaxHeads; h++) a.hc.log2g[h] = 0.0, a.hc.anchor[h] = kChunkAnchorFull;  // shape check only
    pad_small_dk(&a);
    return chunkwise_ws_supported(a) ? chunkwise_scores_bytes(a) : 0;
}

ret_status ret_forward_chunkwise_ws(const void* q, const void* k, const void* v, const double* gammas, int B, int N,
                                    int H, int dk, int dv, int chunk, void* out, float* final_state,
                                    cudaStream_t stream, ret_dtype in_dt, ret_dtype out_dt, int xpos,
                                    int64_t pos_offset, double theta_base, void* workspace, size_t workspace_bytes) {
    t_err[0] = 0;
    RetArgs a;
    ret_status st = make_args(&a, "ret_forward_chunkwise_ws", q, k, v, gammas, B, N, H, dk, dv, chunk, out,
                              final_state, in_dt, out_dt, xpos, pos_offset, theta_base);
    if (st != RET_OK) return st;
    const RetArgs caller = a;
    pad_small_dk(&a);
    const int left = chunkwise_heads_below(a, 0);
    if (!chunkwise_ws_shape_ok(a) || left == H)
        return ret_forward_chunkwise(q, k, v, gammas, B, N, H, dk, dv, chunk, out, final_state, stream, in_dt,
                                     out_dt, xpos, pos_offset, theta_base);
    const size_t need = chunkwise_scores_bytes(a);
    if (!workspace || workspace_bytes < need)
        return fail(RET_ERR_INVALID_ARG, "ret_forward_chunkwise_ws: workspace of %zu bytes needed (got %zu)", need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 256))
        return fail(RET_ERR_INVALID_ARG, "ret_forward_chunkwise_ws: workspace must be 256-byte aligned");
    const size_t ntok = (size_t)B * N * H;
    const size_t bq = ntok * dk * 2, bv = ntok * dv * 2, bo = ntok * dv * (out_dt == RET_F32 ? 4 : 2);
    if (overlaps(workspace, need, q, bq) || overlaps(workspace, need, k, bq) || overlaps(workspace, need, v, bv) ||
        overlaps(workspace, need, out, bo) ||
        (final_state && overlaps(workspace, need, final_state, (size_t)B * H * dk * dv * 4)))
        return fail(RET_ERR_INVALID_ARG, "ret_forward_chunkwise_ws: workspace overlaps another buffer");
    st = launch_chunkwise_scores(a, workspace, stream);
    if (st != RET_OK || left == 0) return st;
    // heads too fast for the tensor-core kernel, token by token
    return launch_recurrent_simt(caller, stream, true);
}

// Workspace checks shared by the workspace-path entry points.
static ret_status check_workspace(const RetArgs& a, const char* who, const void* workspace, size_t workspace_bytes,
                                  bool with_outputs) {
    const size_t need = chunkwise_scores_bytes(a);
    if (!workspace || workspace_bytes < need)
        return fail(RET_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", who, need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 256)) return fail(RET_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    const size_t ntok = (size_t)a.B * a.N * a.H;
    const size_t bq = ntok * dk_of(a) * 2, bv = ntok * a.dv * 2, bo = ntok * a.dv * (a.out_dt == RET_F32 ? 4 : 2);
    const size_t bs = (size_t)a.B * a.H * dk_of(a) * a.dv * 4;
    bool bad = overlaps(workspace, need, a.q, bq) || overlaps(workspace, need, a.k, bq);
    if (with_outputs)
        bad = bad || overlaps(workspace, need, a.v, bv) || overlaps(workspace, need, a.out, bo) ||
              (a.final_state && overlaps(workspace, need, a.final_state, bs)) ||
              (a.initial_state && overlaps(workspace, need, a.initial_state, bs));
    if (bad) return fail(RET_ERR_INVALID_ARG, "%s: workspace overlaps another buffer", who);
    return RET_OK;
}

// initial_state (may be null) against the other buffers of a; final_state
// may be the same buffer.  Sets a->initial_state.
static ret_status check_initial_state(RetArgs* a, const char* who, const float* initial_state) {
    if (!initial_state) return RET_OK;
    const size_t ntok = (size_t)a->B * a->N * a->H, bs = (size_t)a->B * a->H * dk_of(*a) * a->dv * 4;
    const size_t bq = ntok * dk_of(*a) * 2, bv = ntok * a->dv * 2, bo = ntok * a->dv * (a->out_dt == RET_F32 ? 4 : 2);
    if (!aligned(initial_state, 16)) return fail(RET_ERR_INVALID_ARG, "%s: initial_state must be 16-byte aligned", who);
    if (overlaps(initial_state, bs, a->out, bo) || overlaps(initial_state, bs, a->q, bq) ||
        overlaps(initial_state, bs, a->k, bq) || overlaps(initial_state, bs, a->v, bv) ||
        (a->final_state && (const void*)a->final_state != (const void*)initial_state &&
         overlaps(initial_state, bs, a->final_state, bs)))
        return fail(RET_ERR_INVALID_ARG, "%s: initial_state overlaps another buffer (final_state may equal it)", who);
    a->initial_state = initial_state;
    return RET_OK;
}

ret_status ret_chunkwise_prepare(const void* q, const void* k, const double* gammas, int B, int N, int H, int dk,
                                 int dv, int chunk, cudaStream_t stream, ret_dtype in_dt, int xpos,
                                 int64_t pos_offset, double theta_base, void* workspace, size_t workspace_bytes) {
    t_err[0] = 0;
    const char* who = "ret_chunkwise_prepare";
    if (!q || !k) return fail(RET_ERR_INVALID_ARG, "%s: NULL q or k", who);
    if (B < 1 || N < 1 || H < 1 || dk < 1 || dv < 1 || chunk < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
    if (!is_dtype(in_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (xpos && (dk % 2 != 0)) return fail(RET_ERR_INVALID_ARG, "%s: xpos needs an even dk (got %d)", who, dk);
    if (xpos && !(theta_base > 0.0 && isfinite(theta_base)))
        return fail(RET_ERR_INVALID_ARG, "%s: theta_base must be finite and > 0", who);
    if ((size_t)B * N * H * (size_t)(dk > dv ? dk : dv) > ((size_t)1 << 40))
        return fail(RET_ERR_INVALID_ARG, "%s: problem too large", who);
    if (!aligned(q, 16) || !aligned(k, 16)) return fail(RET_ERR_INVALID_ARG, "%s: q, k must be 16-byte aligned", who);
    RetArgs a{};
    a.q = q; a.k = k;
    a.B = B; a.N = N; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk;
    a.in_dt = in_dt; a.out_dt = RET_BF16;
    a.xpos = xpos ? 1 : 0; a.pos_offset = pos_offset; a.theta_base = xpos ? theta_base : 10000.0;
    make_head_consts(gammas, H, &a.hc);
    pad_small_dk(&a);
    if (!chunkwise_ws_supported(a))
        return fail(RET_ERR_UNSUPPORTED, "%s: shape outside the workspace path (ret_chunkwise_workspace_bytes is 0)",
                    who);
    st = check_workspace(a, who, workspace, workspace_bytes, false);
    if (st != RET_OK) return st;
    return launch_chunkwise_scores_pass1(a, workspace, stream);
}

ret_status ret_forward_chunkwise_prepared(const void* q, const void* k, const void* v, const double* gammas, int B,
                                          int N, int H, int dk, int dv, int chunk, void* out, float* final_state,
                                          const float* initial_state, cudaStream_t stream, ret_dtype in_dt,
                                          ret_dtype out_dt, int xpos, int64_t pos_offset, double theta_base,
                                          const void* workspace, size_t workspace_bytes) {
    t_err[0] = 0;
    const char* who = "ret_forward_chunkwise_prepared";
    RetArgs a;
    ret_status st = make_args(&a, who, q, k, v, gammas, B, N, H, dk, dv, chunk, out, final_state, in_dt, out_dt,
                              xpos, pos_offset, theta_base);
    if (st != RET_OK) return st;
    pad_small_dk(&a);
    if (!chunkwise_ws_supported(a))
        return fail(RET_ERR_UNSUPPORTED, "%s: shape outside the workspace path (ret_chunkwise_workspace_bytes is 0)",
                    who);
    st = check_initial_state(&a, who, initial_state);
    if (st != RET_OK) return st;
    st = check_workspace(a, who, workspace, workspace_bytes, true);
    if (st != RET_OK) return st;
    return launch_chunkwise_scores_pass2(a, const_cast<void*>(workspace), stream);
}

size_t ret_normalized_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk, ret_dtype in_dt, int xpos) {
    if (B < 1 || N < 1 || H < 1 || H > kMaxHeads || dk < 1 || dv < 1 || chunk < 1) return 0;
    RetArgs a{};
    a.B = B; a.N = N; a.H = H; a.dk = dk; a.dv = dv; a.chunk = chunk; a.in_dt = in_dt; a.xpos = xpos ? 1 : 0;
    for (int h = 0; h < kMaxHeads; h++) a.hc.log2g[h] = 0.0, a.hc.anchor[h] = kChunkAnchorFull;  // shape check only
    return chunkwise_ws_supported(a) ? normalized_ws_bytes(a) : 0;
}

ret_status ret_forward_chunkwise_normalized(const void* q, const void* k, const void* v, const double* gammas, int B,
                                            int N, int H, int dk, int dv, int chunk, int norm_flags, void* out,
                                            const float* initial_state, float* final_state, const float* initial_z,
                                            float* final_z, cudaStream_t stream, ret_dtype in_dt, ret_dtype out_dt,
                                            int xpos, int64_t pos_offset, double theta_base, void* workspace,
                                            size_t workspace_bytes) {
    t_err[0] = 0;
    const char* who = "ret_forward_chunkwise_normalized";
    RetArgs a;
    ret_status st = make_args(&a, who, q, k, v, gammas, B, N, H, dk, dv, chunk, out, final_state, in_dt, out_dt,
                              xpos, pos_offset, theta_base);
    if (st != RET_OK) return st;
    if (norm_flags & ~(RET_NORM_DECAY | RET_NORM_SCORE))
        return fail(RET_ERR_INVALID_ARG, "%s: norm_flags must combine RET_NORM_DECAY and RET_NORM_SCORE", who);
    if (pos_offset < 0) return fail(RET_ERR_INVALID_ARG, "%s: pos_offset must be >= 0", who);
    if (!chunkwise_ws_supported(a) || chunkwise_heads_below(a, kChunkAnchorFull) > 0)
        return fail(RET_ERR_UNSUPPORTED,
                    "%s: needs bf16 inputs, chunk 128, dk 128 or 256, dv a multiple of 64 and every "
                    "gamma_h^128 >= 2^-60",
                    who);
    st = check_initial_state(&a, who, initial_state);
    if (st != RET_OK) return st;
    const size_t ntok = (size_t)B * N * H, bz = (size_t)B * H * dk * 4, bs = (size_t)B * H * dk * dv * 4;
    const size_t bq = ntok * dk * 2, bv = ntok * dv * 2, bo = ntok * dv * (out_dt == RET_F32 ? 4 : 2);
    for (const float* z : {initial_z, (const float*)final_z}) {
        if (!z) continue;
        if (!aligned(z, 16)) return fail(RET_ERR_INVALID_ARG, "%s: initial_z and final_z must be 16-byte aligned", who);
        if (overlaps(z, bz, q, bq) || overlaps(z, bz, k, bq) || overlaps(z, bz, v, bv) || overlaps(z, bz, out, bo) ||
            (final_state && overlaps(z, bz, final_state, bs)) || (initial_state && overlaps(z, bz, initial_state, bs)))
            return fail(RET_ERR_INVALID_ARG, "%s: initial_z or final_z overlaps another buffer", who);
    }
    if (initial_z && final_z && initial_z != final_z && overlaps(initial_z, bz, final_z, bz))
        return fail(RET_ERR_INVALID_ARG, "%s: initial_z and final_z overlap (they may be the same buffer)", who);
    const size_t need = normalized_ws_bytes(a);
    if (!workspace || workspace_bytes < need)
        return fail(RET_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", who, need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 256)) return fail(RET_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    if (overlaps(workspace, need, q, bq) || overlaps(workspace, need, k, bq) || overlaps(workspace, need, v, bv) ||
        overlaps(workspace, need, out, bo) || (final_state && overlaps(workspace, need, final_state, bs)) ||
        (initial_state && overlaps(workspace, need, initial_state, bs)) ||
        (initial_z && overlaps(workspace, need, initial_z, bz)) || (final_z && overlaps(workspace, need, final_z, bz)))
        return fail(RET_ERR_INVALID_ARG, "%s: workspace overlaps another buffer", who);
    return launch_chunkwise_normalized(a, norm_flags, initial_z, final_z, workspace, stream);
}

static void fill_bwd(BwdArgs* b, const void* q, const void* k, const void* v, const void* dout, int B, int N, int H,
                     int dk, int dv, int chunk, int xpos, int64_t pos_offset, double theta_base) {
    memset(b, 0, sizeof(*b));
    b->q = q; b->k = k; b->v = v; b->dout = dout;
    b->B = B; b->N = N; b->H = H; b->dk = dk; b->dv = dv; b->chunk = chunk;
    b->xpos = xpos ? 1 : 0; b->pos_offset = pos_offset; b->theta_base = xpos ? theta_base : 10000.0;
}

size_t ret_backward_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk, ret_dtype in_dt, int xpos) {
    if (B < 1 || N < 1 || H < 1 || H > kMaxHeads || dk < 1 || dv < 1 || chunk < 1 || in_dt != RET_BF16) return 0;
    BwdArgs b;
    fill_bwd(&b, nullptr, nullptr, nullptr, nullptr, B, N, H, dk, dv, chunk, xpos, 0, 10000.0);
    return backward_supported(b) ? backward_ws_bytes(b) : 0;
}

ret_status ret_backward_chunkwise(const void* q, const void* k, const void* v, const void* dout,
                                  const double* gammas, int B, int N, int H, int dk, int dv, int chunk, float* dq,
                                  float* dk_out, float* dv_out, cudaStream_t stream, ret_dtype in_dt, int xpos,
                                  int64_t pos_offset, double theta_base, void* workspace, size_t workspace_bytes) {
    t_err[0] = 0;
    const char* who = "ret_backward_chunkwise";
    if (!q || !k || !v || !dout || !dq || !dk_out || !dv_out)
        return fail(RET_ERR_INVALID_ARG, "%s: NULL q, k, v, dout, dq, dk or dv", who);
    if (B < 1 || N < 1 || H < 1 || dk < 1 || dv < 1 || chunk < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
    if (!is_dtype(in_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (xpos && (dk % 2 != 0)) return fail(RET_ERR_INVALID_ARG, "%s: xpos needs an even dk", who);
    if (xpos && !(theta_base > 0.0 && isfinite(theta_base)))
        return fail(RET_ERR_INVALID_ARG, "%s: theta_base must be finite and > 0", who);
    if ((size_t)B * N * H * (size_t)(dk > dv ? dk : dv) > ((size_t)1 << 40))
        return fail(RET_ERR_INVALID_ARG, "%s: problem too large", who);
    for (const void* p : {q, k, v, dout, (const void*)dq, (const void*)dk_out, (const void*)dv_out})
        if (!aligned(p, 16)) return fail(RET_ERR_INVALID_ARG, "%s: device pointers must be 16-byte aligned", who);
    BwdArgs b;
    fill_bwd(&b, q, k, v, dout, B, N, H, dk, dv, chunk, xpos, pos_offset, theta_base);
    b.dq = dq; b.dkk = dk_out; b.dvv = dv_out;
    make_head_consts(gammas, H, &b.hc);
    if (in_dt != RET_BF16 || !backward_supported(b))
        return fail(RET_ERR_UNSUPPORTED,
                    "%s: needs bf16 inputs, chunk 128, dk 128 or 256, dv a multiple of 128 and every "
                    "gamma_h^128 >= 2^-60",
                    who);
    const size_t need = backward_ws_bytes(b);
    if (!workspace || workspace_bytes < need)
        return fail(RET_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", who, need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 256)) return fail(RET_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    const size_t ntok = (size_t)B * N * H;
    const size_t bq = ntok * dk * 2, bv = ntok * dv * 2, gq = ntok * dk * 4, gv = ntok * dv * 4;
    const void* ins[4] = {q, k, v, dout};
    const size_t insz[4] = {bq, bq, bv, bv};
    const void* outs[3] = {dq, dk_out, dv_out};
    const size_t outsz[3] = {gq, gq, gv};
    for (int i = 0; i < 3; i++) {
        if (overlaps(outs[i], outsz[i], workspace, need))
            return fail(RET_ERR_INVALID_ARG, "%s: an output overlaps the workspace", who);
        for (int j = 0; j < 4; j++)
            if (overlaps(outs[i], outsz[i], ins[j], insz[j]))
                return fail(RET_ERR_INVALID_ARG, "%s: an output overlaps an input", who);
        for (int j = i + 1; j < 3; j++)
            if (overlaps(outs[i], outsz[i], outs[j], outsz[j]))
                return fail(RET_ERR_INVALID_ARG, "%s: outputs overlap", who);
    }
    for (int j = 0; j < 4; j++)
        if (overlaps(workspace, need, ins[j], insz[j]))
            return fail(RET_ERR_INVALID_ARG, "%s: workspace overlaps an input", who);
    b.workspace = workspace;
    return launch_backward(b, stream);
}

ret_status ret_forward_chunkwise_noalloc(const void* q, const void* k, const void* v, const double* gammas, int B,
                                         int N, int H, int dk, int dv, int chunk, void* out, float* final_state,
                                         cudaStream_t stream, ret_dtype in_dt, ret_dtype out_dt, int xpos,
                                         int64_t pos_offset, double theta_base) {
    t_err[0] = 0;
    RetArgs a;
    ret_status st = make_args(&a, "ret_forward_chunkwise_noalloc", q, k, v, gammas, B, N, H, dk, dv, chunk, out,
                              final_state, in_dt, out_dt, xpos, pos_offset, theta_base);
    if (st != RET_OK) return st;
    pad_small_dk(&a);
    if (!chunkwise_ws_supported(a))
        return fail(RET_ERR_UNSUPPORTED,
                    "ret_forward_chunkwise_noalloc: needs bf16 inputs, chunk 128, dk 128 or 256, dv a multiple of "
                    "64 and every gamma_h^64 >= 2^-100");
    return launch_chunkwise_static(a, stream);
}

size_t ret_chunkwise_noalloc_max_bytes(void) { return chunkwise_static_ws_bytes(); }

ret_status ret_forward_parallel(const void* q, const void* k, const void* v, const double* gammas, int B, int N,
                                int H, int dk, int dv, void* out, cudaStream_t stream, ret_dtype in_dt,
                                ret_dtype out_dt, int xpos, int64_t pos_offset, double theta_base) {
    t_err[0] = 0;
    RetArgs a;
    ret_status st = make_args(&a, "ret_forward_parallel", q, k, v, gammas, B, N, H, dk, dv, 1, out, nullptr,
                              in_dt, out_dt, xpos, pos_offset, theta_base);
    if (st != RET_OK) return st;
    return launch_parallel_simt(a, stream);
}

ret_status ret_forward_recurrent(const void* q, const void* k, const void* v, const double* gammas, int B, int N,
                                 int H, int dk, int dv, void* out, float* final_state, cudaStream_t stream,
                                 ret_dtype in_dt, ret_dtype out_dt, int xpos, int64_t pos_offset,
                                 double theta_base) {
    t_err[0] = 0;
    RetArgs a;
    ret_status st = make_args(&a, "ret_forward_recurrent", q, k, v, gammas, B, N, H, dk, dv, 1, out,
                              final_state, in_dt, out_dt, xpos, pos_offset, theta_base);
    if (st != RET_OK) return st;
    return launch_recurrent_simt(a, stream);
}

ret_status ret_decode_step(const void* q, const void* k, const void* v, const double* gammas, float* state,
                           void* out, cudaStream_t stream, int B, int H, int dk, int dv, ret_dtype in_dt,
                           ret_dtype out_dt) {
    t_err[0] = 0;
    const char* who = "ret_decode_step";
    if (!q || !k || !v || !state || !out) return fail(RET_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
    if (B < 1 || H < 1 || dk < 1 || dv < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1 (B=%d H=%d dk=%d dv=%d)", who, B, H, dk, dv);
    if (!is_dtype(in_dt) || !is_dtype(out_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (dv % 4 != 0) return fail(RET_ERR_INVALID_ARG, "%s: dv must be a multiple of 4 (got %d)", who, dv);
    if (!aligned(state, 16)) return fail(RET_ERR_INVALID_ARG, "%s: state must be 16-byte aligned", who);
    for (const void* p : {q, k, v, (const void*)out})
        if (!aligned(p, 4)) return fail(RET_ERR_INVALID_ARG, "%s: q, k, v, out must be 4-byte aligned", who);
    const size_t bs = (size_t)B * H * dk * dv * 4, bo = (size_t)B * H * dv * esize(out_dt);
    if (overlaps(out, bo, state, bs)) return fail(RET_ERR_INVALID_ARG, "%s: out overlaps state", who);
    HeadConsts hc;
    make_head_consts(gammas, H, &hc);
    return launch_decode(q, k, v, hc, state, out, B, H, dk, dv, in_dt, out_dt, stream);
}

ret_status ret_decode_step_normalized(const void* q, const void* k, const void* v, const double* gammas,
                                      float* state, float* z, void* out, int64_t position, int norm_flags,
                                      cudaStream_t stream, int B, int H, int dk, int dv, ret_dtype in_dt,
                                      ret_dtype out_dt) {
    t_err[0] = 0;
    const char* who = "ret_decode_step_normalized";
    if (!q || !k || !v || !state || !out) return fail(RET_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
    if (B < 1 || H < 1 || dk < 1 || dv < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1 (B=%d H=%d dk=%d dv=%d)", who, B, H, dk, dv);
    if (!is_dtype(in_dt) || !is_dtype(out_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (norm_flags & ~(RET_NORM_DECAY | RET_NORM_SCORE))
        return fail(RET_ERR_INVALID_ARG, "%s: norm_flags must combine RET_NORM_DECAY and RET_NORM_SCORE", who);
    if ((norm_flags & RET_NORM_SCORE) && !z)
        return fail(RET_ERR_INVALID_ARG, "%s: RET_NORM_SCORE needs the key-sum state z", who);
    if (position < 0) return fail(RET_ERR_INVALID_ARG, "%s: position must be >= 0", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (dv % 4 != 0) return fail(RET_ERR_INVALID_ARG, "%s: dv must be a multiple of 4 (got %d)", who, dv);
    if (!aligned(state, 16)) return fail(RET_ERR_INVALID_ARG, "%s: state must be 16-byte aligned", who);
    for (const void* p : {q, k, v, (const void*)out})
        if (!aligned(p, 4)) return fail(RET_ERR_INVALID_ARG, "%s: q, k, v, out must be 4-byte aligned", who);
    const size_t bs = (size_t)B * H * dk * dv * 4, bo = (size_t)B * H * dv * esize(out_dt);
    const size_t bz = (size_t)B * H * dk * 4, bq = (size_t)B * H * dk * esize(in_dt);
    if (overlaps(out, bo, state, bs)) return fail(RET_ERR_INVALID_ARG, "%s: out overlaps state", who);
    if (z && (norm_flags & RET_NORM_SCORE)) {
        if (!aligned(z, 16)) return fail(RET_ERR_INVALID_ARG, "%s: z must be 16-byte aligned", who);
        if (overlaps(z, bz, state, bs) || overlaps(z, bz, out, bo) || overlaps(z, bz, q, bq) || overlaps(z, bz, k, bq))
            return fail(RET_ERR_INVALID_ARG, "%s: z overlaps another buffer", who);
    }
    HeadConsts hc;
    make_head_consts(gammas, H, &hc);
    DecodeOpts o{};
    o.z = (norm_flags & RET_NORM_SCORE) ? z : nullptr;
    o.pos = position;
    o.flags = norm_flags;
    return launch_decode_ex(q, k, v, hc, state, out, B, H, dk, dv, in_dt, out_dt, o, stream);
}

ret_status ret_decode_step_positions(const void* q, const void* k, const void* v, const double* gammas,
                                     float* state, float* z, void* out, const int64_t* positions, int xpos,
                                     double theta_base, int norm_flags, cudaStream_t stream, int B, int H, int dk,
                                     int dv, ret_dtype in_dt, ret_dtype out_dt) {
    t_err[0] = 0;
    const char* who = "ret_decode_step_positions";
    if (!q || !k || !v || !state || !out || !positions)
        return fail(RET_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
    if (B < 1 || H < 1 || dk < 1 || dv < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1 (B=%d H=%d dk=%d dv=%d)", who, B, H, dk, dv);
    if (!is_dtype(in_dt) || !is_dtype(out_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (norm_flags & ~(RET_NORM_DECAY | RET_NORM_SCORE))
        return fail(RET_ERR_INVALID_ARG, "%s: norm_flags must combine RET_NORM_DECAY and RET_NORM_SCORE", who);
    if ((norm_flags & RET_NORM_SCORE) && !z)
        return fail(RET_ERR_INVALID_ARG, "%s: RET_NORM_SCORE needs the key-sum state z", who);
    if (xpos && dk % 2) return fail(RET_ERR_INVALID_ARG, "%s: xpos needs an even dk (got %d)", who, dk);
    if (xpos && !(theta_base > 0.0 && isfinite(theta_base)))
        return fail(RET_ERR_INVALID_ARG, "%s: theta_base must be finite and > 0", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (dv % 4 != 0) return fail(RET_ERR_INVALID_ARG, "%s: dv must be a multiple of 4 (got %d)", who, dv);
    if (!aligned(state, 16)) return fail(RET_ERR_INVALID_ARG, "%s: state must be 16-byte aligned", who);
    if (!aligned(positions, 8)) return fail(RET_ERR_INVALID_ARG, "%s: positions must be 8-byte aligned", who);
    for (const void* p : {q, k, v, (const void*)out})
        if (!aligned(p, 4)) return fail(RET_ERR_INVALID_ARG, "%s: q, k, v, out must be 4-byte aligned", who);
    const size_t bs = (size_t)B * H * dk * dv * 4, bo = (size_t)B * H * dv * esize(out_dt);
    const size_t bz = (size_t)B * H * dk * 4, bq = (size_t)B * H * dk * esize(in_dt);
    if (overlaps(out, bo, state, bs)) return fail(RET_ERR_INVALID_ARG, "%s: out overlaps state", who);
    if (overlaps(positions, (size_t)B * 8, state, bs) || overlaps(positions, (size_t)B * 8, out, bo))
        return fail(RET_ERR_INVALID_ARG, "%s: positions overlap another buffer", who);
    if (z && (norm_flags & RET_NORM_SCORE)) {
        if (!aligned(z, 16)) return fail(RET_ERR_INVALID_ARG, "%s: z must be 16-byte aligned", who);
        if (overlaps(z, bz, state, bs) || overlaps(z, bz, out, bo) || overlaps(z, bz, q, bq) ||
            overlaps(z, bz, k, bq) || overlaps(z, bz, positions, (size_t)B * 8))
            return fail(RET_ERR_INVALID_ARG, "%s: z overlaps another buffer", who);
    }
    HeadConsts hc;
    make_head_consts(gammas, H, &hc);
    DecodeOpts o{};
    o.z = (norm_flags & RET_NORM_SCORE) ? z : nullptr;
    o.positions = reinterpret_cast<const long long*>(positions);
    o.flags = norm_flags;
    o.xpos = xpos ? 1 : 0;
    o.log2base = log2(xpos ? theta_base : 10000.0);
    return launch_decode_ex(q, k, v, hc, state, out, B, H, dk, dv, in_dt, out_dt, o, stream);
}

size_t ret_msr_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv) {
    if (B < 1 || N < 1 || dmodel < 1 || H < 1 || dk < 1 || dv < 1) return 0;
    return msr_workspace_bytes(B, N, dmodel, H, dk, dv);
}

ret_status ret_msr_forward(const void* X, const void* Wq, const void* Wk, const void* Wv, const void* Wg,
                           const void* Wo, const double* gammas, int B, int N, int dmodel, int H, int dk, int dv,
                           int chunk, double k_scale, double eps, int xpos, int64_t pos_offset, double theta_base,
                           void* out, ret_dtype out_dt, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    t_err[0] = 0;
    const char* who = "ret_msr_forward";
    for (const void* ptr : {X, Wq, Wk, Wv, Wg, Wo, (const void*)out, (const void*)workspace})
        if (!ptr) return fail(RET_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
    for (const void* ptr : {X, Wq, Wk, Wv, Wg, Wo, (const void*)out})
        if (!aligned(ptr, 16)) return fail(RET_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    if (!aligned(workspace, 256)) return fail(RET_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    if (B < 1 || N < 1 || dmodel < 1 || H < 1 || dk < 1 || dv < 1 || chunk < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
    if (!is_dtype(out_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (dmodel % 8) return fail(RET_ERR_INVALID_ARG, "%s: d_model must be a multiple of 8", who);
    if (!(eps >= 0.0) || !isfinite(k_scale)) return fail(RET_ERR_INVALID_ARG, "%s: bad eps or k_scale", who);
    if (xpos && !(theta_base > 0.0 && isfinite(theta_base)))
        return fail(RET_ERR_INVALID_ARG, "%s: theta_base must be finite and > 0", who);
    const size_t need = msr_workspace_bytes(B, N, dmodel, H, dk, dv);
    if (workspace_bytes < need)
        return fail(RET_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", who, need, workspace_bytes);
    const size_t M = (size_t)B * N;
    const size_t bx = M * dmodel * 2, bo = M * dmodel * (out_dt == RET_F32 ? 4 : 2);
    if (overlaps(out, bo, X, bx) || overlaps(workspace, need, X, bx) || overlaps(workspace, need, out, bo))
        return fail(RET_ERR_INVALID_ARG, "%s: out or workspace overlaps another buffer", who);
    MsrArgs m;
    m.X = X; m.Wq = Wq; m.Wk = Wk; m.Wv = Wv; m.Wg = Wg; m.Wo = Wo;
    m.B = B; m.N = N; m.dmodel = dmodel; m.H = H; m.dk = dk; m.dv = dv; m.chunk = chunk;
    m.k_scale = k_scale; m.eps = eps; m.xpos = xpos ? 1 : 0; m.pos_offset = pos_offset;
    m.theta_base = xpos ? theta_base : 10000.0;
    make_head_consts(gammas, H, &m.hc);
    m.out = out; m.out_dt = out_dt; m.workspace = workspace; m.residual = nullptr;
    // the retention step runs on the tensor-core kernel only
    RetArgs a{};
    a.B = B; a.in_dt = RET_BF16; a.chunk = chunk; a.dk = dk; a.dv = dv; a.N = N; a.H = H; a.hc = m.hc;
    // (the projection epilogue scales the keys by the plain zeta)
    if (!chunkwise_ws_supported(a) || chunkwise_heads_below(a, kChunkAnchorFull) > 0)
        return fail(RET_ERR_UNSUPPORTED, "%s: needs chunk 128, d_k 128 or 256, d_v a multiple of 64 and "
                    "gamma_h^128 >= 2^-60", who);
    if (!(dv == 128 || dv == 256 || dv == 512 || dv == 1024))
        return fail(RET_ERR_UNSUPPORTED, "%s: d_v must be 128, 256, 512 or 1024", who);
    return launch_msr(m, stream);
}

size_t ret_retnet_block_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv, int dff) {
    if (B < 1 || N < 1 || dmodel < 1 || H < 1 || dk < 1 || dv < 1 || dff < 1) return 0;
    return block_workspace_bytes(B, N, dmodel, H, dk, dv, dff);
}

ret_status ret_retnet_block_forward(const void* X, const void* ln1_gain, const void* ln1_bias, const void* Wq,
                                    const void* Wk, const void* Wv, const void* Wg, const void* Wo,
                                    const void* ln2_gain, const void* ln2_bias, const void* W1, const void* W2,
                                    const double* gammas, int B, int N, int dmodel, int H, int dk, int dv, int dff,
                                    int chunk, double k_scale, double gn_eps, double ln_eps, int xpos,
                                    int64_t pos_offset, double theta_base, void* out, ret_dtype out_dt,
                                    void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    t_err[0] = 0;
    const char* who = "ret_retnet_block_forward";
    for (const void* ptr : {X, Wq, Wk, Wv, Wg, Wo, W1, W2, (const void*)out, (const void*)workspace})
        if (!ptr) return fail(RET_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
    for (const void* ptr : {X, Wq, Wk, Wv, Wg, Wo, W1, W2, (const void*)out})
        if (!aligned(ptr, 16)) return fail(RET_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    for (const void* ptr : {ln1_gain, ln1_bias, ln2_gain, ln2_bias})
        if (ptr && !aligned(ptr, 4)) return fail(RET_ERR_INVALID_ARG, "%s: LayerNorm parameters must be 4-byte aligned", who);
    if (!aligned(workspace, 256)) return fail(RET_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", who);
    if (B < 1 || N < 1 || dmodel < 1 || H < 1 || dk < 1 || dv < 1 || dff < 1 || chunk < 1)
        return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
    if (!is_dtype(out_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    ret_status st = check_gammas(gammas, H, who);
    if (st != RET_OK) return st;
    if (dmodel % 8 || dff % 8) return fail(RET_ERR_INVALID_ARG, "%s: d_model and d_ff must be multiples of 8", who);
    if (!(gn_eps >= 0.0) || !(ln_eps >= 0.0) || !isfinite(k_scale))
        return fail(RET_ERR_INVALID_ARG, "%s: bad eps or k_scale", who);
    if (xpos && !(theta_base > 0.0 && isfinite(theta_base)))
        return fail(RET_ERR_INVALID_ARG, "%s: theta_base must be finite and > 0", who);
    const size_t need = block_workspace_bytes(B, N, dmodel, H, dk, dv, dff);
    if (workspace_bytes < need)
        return fail(RET_ERR_INVALID_ARG, "%s: workspace of %zu bytes needed (got %zu)", who, need, workspace_bytes);
    const size_t M = (size_t)B * N;
    const size_t bx = M * dmodel * 2, bo = M * dmodel * (out_dt == RET_F32 ? 4 : 2);
    if (overlaps(out, bo, X, bx) || overlaps(workspace, need, X, bx) || overlaps(workspace, need, out, bo))
        return fail(RET_ERR_INVALID_ARG, "%s: out or workspace overlaps another buffer", who);
    RetArgs a{};
    a.B = B; a.in_dt = RET_BF16; a.chunk = chunk; a.dk = dk; a.dv = dv; a.N = N; a.H = H;
    make_head_consts(gammas, H, &a.hc);
    if (!chunkwise_ws_supported(a) || chunkwise_heads_below(a, kChunkAnchorFull) > 0)
        return fail(RET_ERR_UNSUPPORTED, "%s: needs chunk 128, d_k 128 or 256, d_v a multiple of 64 and "
                    "gamma_h^128 >= 2^-60", who);
    if (!(dv == 128 || dv == 256 || dv == 512 || dv == 1024))
        return fail(RET_ERR_UNSUPPORTED, "%s: d_v must be 128, 256, 512 or 1024", who);
    BlockArgs b;
    memset(&b, 0, sizeof(b));
    MsrArgs& m = b.msr;
    m.X = X; m.Wq = Wq; m.Wk = Wk; m.Wv = Wv; m.Wg = Wg; m.Wo = Wo;
    m.B = B; m.N = N; m.dmodel = dmodel; m.H = H; m.dk = dk; m.dv = dv; m.chunk = chunk;
    m.k_scale = k_scale; m.eps = gn_eps; m.xpos = xpos ? 1 : 0; m.pos_offset = pos_offset;
    m.theta_base = xpos ? theta_base : 10000.0;
    m.hc = a.hc;
    b.ln1_g = ln1_gain; b.ln1_b = ln1_bias; b.ln2_g = ln2_gain; b.ln2_b = ln2_bias;
    b.W1 = W1; b.W2 = W2; b.dff = dff; b.ln_eps = ln_eps;
    b.out = out; b.out_dt = out_dt; b.workspace = workspace;
    return launch_block(b, stream);
}

ret_status ret_linear_bf16(const void* X, const void* W, void* Y, int M, int N, int K, ret_dtype out_dt,
                           cudaStream_t stream) {
    t_err[0] = 0;
    const char* who = "ret_linear_bf16";
    if (!X || !W || !Y) return fail(RET_ERR_INVALID_ARG, "%s: NULL pointer argument", who);
    if (M < 1 || N < 1 || K < 1) return fail(RET_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
    if (N % 8 || K % 8) return fail(RET_ERR_INVALID_ARG, "%s: N and K must be multiples of 8", who);
    if (!is_dtype(out_dt)) return fail(RET_ERR_INVALID_ARG, "%s: unknown dtype", who);
    for (const void* ptr : {X, W, (const void*)Y})
        if (!aligned(ptr, 16)) return fail(RET_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
    const size_t by = (size_t)M * N * (out_dt == RET_F32 ? 4 : 2);
    if (overlaps(Y, by, X, (size_t)M * K * 2) || overlaps(Y, by, W, (size_t)K * N * 2))
        return fail(RET_ERR_INVALID_ARG, "%s: Y overlaps an input", who);
    return launch_linear(X, W, Y, M, N, K, out_dt, stream);
}

ret_status ret_selftest_bounded_wait(uint32_t polls, cudaStream_t stream) {
    t_err[0] = 0;
    if (polls < 1 || polls > (1u << 24))
        return fail(RET_ERR_INVALID_ARG, "ret_selftest_bounded_wait: polls must be in [1, 2^24]");
    return launch_wait_selftest(polls, stream);
}

ret_status ret_check_device_error(cudaStream_t stream) {
    t_err[0] = 0;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "ret_check_device_error: %s", cudaGetErrorString(e));
    int flag = 0, flag2 = 0;
    e = read_clear_error_chunk_ws(&flag);
    if (e == cudaSuccess) e = read_clear_error_gemm(&flag2);
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "ret_check_device_error: %s", cudaGetErrorString(e));
    flag |= flag2;
    if (flag) return fail(RET_ERR_TIMEOUT, "a kernel gave up a bounded wait (device error word %d)", flag);
    return RET_OK;
}

}  // extern "C"
