// kernels.h -- internal launch functions behind the C ABI.  Each returns
// RET_OK after enqueueing, RET_ERR_UNSUPPORTED if the shape does not fit the
// kernel (nothing launched), or RET_ERR_CUDA if the launch failed.  Argument
// validation has already happened in ret_api.cu.
#pragma once

#include "common.cuh"

namespace ret {

struct RetArgs {
    const void* q;
    const void* k;
    const void* v;
    void* out;
    float* final_state;          // may be null
    const float* initial_state;  // may be null (zero state); workspace path only
    // Workspace path only: elements between consecutive (token, head) rows of
    // q and of k (0: dk, i.e. contiguous), so that a column slice of a wider
    // tensor can serve as q or k; accumulate = 1 adds the result into an
    // fp32 out instead of storing it; out_rev = 1 writes the output of token n
    // to row N-1-n.
    int q_ld, k_ld, accumulate, out_rev;
    // Workspace path only: fp32 [B, N, H] factors the output row of each
    // (token, head) is multiplied by (the score normalizations), or null.
    const float* rowscale;
    // Workspace path only: the caller's d_k when it is below the tensor-core
    // kernel's (0: dk).  The rows are then zero-padded to dk in the
    // workspace, the rotation uses dk_real, and the states have dk_real rows.
    int dk_real;
    int B, N, H, dk, dv, chunk;
    ret_dtype in_dt, out_dt;
    int xpos;
    long long pos_offset;
    double theta_base;
    HeadConsts hc;
    double gamma[kMaxHeads];
};

// inverse: turn by -angle (the transpose of each rotation).
ret_status launch_xpos_rotate(void* x, ret_dtype dt, int B, int N, int H, int d, long long pos_offset,
                              double theta_base, cudaStream_t s, bool inverse = false);
ret_status launch_chunkwise_simt(const RetArgs& a, cudaStream_t s);
ret_status launch_parallel_simt(const RetArgs& a, cudaStream_t s);
// untaken_only: only the heads the tensor-core kernels leave out (anchor -1).
ret_status launch_recurrent_simt(const RetArgs& a, cudaStream_t s, bool untaken_only = false);
ret_status launch_decode(const void* q, const void* k, const void* v, const HeadConsts& hc, float* state,
                         void* out, int B, int H, int dk, int dv, ret_dtype in_dt, ret_dtype out_dt,
                         cudaStream_t s);


// Workspace path: prep kernel (rotation + zeta scaling into the workspace)
// and the warp-specialized tensor-core kernel.  The shape check alone; the
// number of heads whose anchor (HeadConsts) is below min_anchor (0: heads the
// kernel does not take; kChunkAnchorFull: heads not on the plain factors);
// and both together (shape on the path, every head taken).
bool chunkwise_ws_shape_ok(const RetArgs& a);
int chunkwise_heads_below(const RetArgs& a, int min_anchor);
bool chunkwise_ws_supported(const RetArgs& a);
size_t chunkwise_ws_bytes(const RetArgs& a);
ret_status launch_chunkwise_ws(const RetArgs& a, void* ws, cudaStream_t s);
// Its two halves: the prep pass alone, and the tensor-core kernel on a
// workspace the prep pass has filled (a.initial_state honoured).
ret_status launch_chunkwise_prep(const RetArgs& a, void* ws, cudaStream_t s);
ret_status launch_chunkwise_prepared(const RetArgs& a, void* ws, cudaStream_t s);
// The scores form: a tensor-core pass that rotates q and k, scales the keys
// and computes the masked intra-chunk scores P of every (b, h, chunk), then
// the warp-specialized kernel on those (read-out, P V, state update).  `ws`
// holds chunkwise_scores_bytes (256-byte aligned).  The pooled form takes it
// from a stream-ordered pool of the library.
size_t chunkwise_scores_bytes(const RetArgs& a);
ret_status launch_chunkwise_scores(const RetArgs& a, void* ws, cudaStream_t s);
// Its two passes on their own (the second honours a.initial_state).
ret_status launch_chunkwise_scores_pass1(const RetArgs& a, void* ws, cudaStream_t s);
ret_status launch_chunkwise_scores_pass2(const RetArgs& a, void* ws, cudaStream_t s);
ret_status launch_chunkwise_scores_pooled(const RetArgs& a, cudaStream_t s);
// The workspace path on the library's fixed device array (no allocation).
size_t chunkwise_static_ws_bytes();
ret_status launch_chunkwise_static(const RetArgs& a, cudaStream_t s);
// Score normalizations 2 and 3 on the workspace path: flags bit 0 divides
// row n of the decay matrix by sqrt(sum_i D_ni), bit 1 the scores by
// max(|sum_i R_ni|, 1); z0 / z1 the decayed key sum before / after the
// call ([B, H, dk] fp32, either may be null).
constexpr int kNormDecay = RET_NORM_DECAY, kNormScore = RET_NORM_SCORE;
size_t normalized_ws_bytes(const RetArgs& a);
ret_status launch_chunkwise_normalized(const RetArgs& a, int flags, const float* z0, float* z1, void* ws,
                                       cudaStream_t s);
// Options of the decode step: the xPos rotation of q and k and the score
// normalizations at each sequence's position (positions[b] on the device, or
// pos for all when positions is null); z [B, H, dk] updated in place (needed
// with kNormScore).
struct DecodeOpts {
    float* z;
    const long long* positions;
    long long pos;
    int flags;
    int xpos;
    double log2base;
};
ret_status launch_decode_ex(const void* q, const void* k, const void* v, const HeadConsts& hc, float* state,
                            void* out, int B, int H, int dk, int dv, ret_dtype in_dt, ret_dtype out_dt,
                            const DecodeOpts& o, cudaStream_t s);

// One thread waits on a barrier nothing arrives on (bounded), then sets the
// device error word: the timeout path without a hang or a fault.
ret_status launch_wait_selftest(uint32_t polls, cudaStream_t s);

// The tensor-core kernel alone, on prepared q_rot (or q) and k' (zeta-scaled keys).
// q_rot: [B, N, H, dk] rows q_pitch elements apart.
ret_status launch_chunkwise_main(const RetArgs& a, const void* q_rot, int q_pitch, const void* k_prime,
                                 cudaStream_t s);

// Gradients of chunkwise retention (k_backward.cu): bf16 q, k, v, dout
// [B, N, H, d], fp32 dq, dk, dv.
struct BwdArgs {
    const void *q, *k, *v, *dout;
    float *dq, *dkk, *dvv;
    int B, N, H, dk, dv, chunk;
    int xpos;
    long long pos_offset;
    double theta_base;
    HeadConsts hc;
    void* workspace;
};
bool backward_supported(const BwdArgs& a);
size_t backward_ws_bytes(const BwdArgs& a);
ret_status launch_backward(const BwdArgs& a, cudaStream_t s);

struct MsrArgs {
    const void *X, *Wq, *Wk, *Wv, *Wg, *Wo;
    int B, N, dmodel, H, dk, dv, chunk;
    double k_scale, eps;
    int xpos;
    long long pos_offset;
    double theta_base;
    HeadConsts hc;
    void* out;
    ret_dtype out_dt;
    void* workspace;
    const void* residual;  // bf16 [B*N, dmodel] added to the output, or null
};
size_t msr_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv);
ret_status launch_msr(const MsrArgs& m, cudaStream_t s);
ret_status launch_linear(const void* X, const void* W, void* Y, int M, int N, int K, ret_dtype out_dt, cudaStream_t s);

// One pre-norm RetNet block: Y = MSR(LN1(X)) + X, out = gelu(LN2(Y) W1) W2 + Y.
struct BlockArgs {
    MsrArgs msr;            // X, the MSR weights and shapes; out / residual / workspace unused
    const void *ln1_g, *ln1_b, *ln2_g, *ln2_b;  // bf16 [dmodel] each, or null (gain 1, bias 0)
    const void *W1, *W2;    // bf16 [dmodel, dff], [dff, dmodel]
    int dff;
    double ln_eps;
    void* out;
    ret_dtype out_dt;
    void* workspace;
};
size_t block_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv, int dff);
ret_status launch_block(const BlockArgs& a, cudaStream_t s);
// LayerNorm of the rows of x [M, d] (bf16) into y (bf16).
ret_status launch_layernorm(const void* x, const void* gain, const void* bias, void* y, int M, int d, double eps,
                            cudaStream_t s);

}  // namespace ret
