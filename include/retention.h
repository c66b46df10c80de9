/*
 * retention.h -- C ABI of the B200 (sm_100a) multi-scale retention library.
 *
 * The library computes retention, the sequence mixer of the Retentive Network:
 *     o_n = sum_{m <= n} gamma_h^(n-m) (q_n . k_m) v_m        (per head h)
 * defined by the recurrence S_n = gamma S_{n-1} + k_n v_n^T, o_n = q_n^T S_n
 * ("Hybrid Architectures: RetNet and the Three Computation Paradigms",
 * sections 2.1-2.2; RetNet paper summary, Eq. 6).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  Row-major, last index fastest:
 *     q, k          [B, N, H, dk]      (decode: [B, H, dk])
 *     v, out        [B, N, H, dv]      (decode: [B, H, dv])
 *     state         [B, H, dk, dv]     always fp32
 * Positions are 0-based: token n sits at position pos_offset + n.
 *
 * Dtypes.  RET_BF16 inputs are multiplied in the tensor cores with fp32
 * accumulation; RET_F32 inputs run on the CUDA cores in fp32 (no TF32).
 * Every carried state is fp32.
 *
 * gammas.  A HOST pointer to H doubles, each in [0, 1].  The library turns
 * them into per-head constants on the host in fp64 and passes those by value
 * to the kernels, so the array may be freed as soon as the call returns.
 *
 * Ownership.  The caller allocates every device buffer.  The library keeps
 * no pointer after a call returns and allocates nothing, except where an
 * entry point says so.
 *
 * Asynchrony.  Every call enqueues its kernels on `stream` and returns
 * without synchronising.  Results are valid once the stream has completed.
 * Calls are thread-safe; the error string is per thread.
 *
 * Errors.  Every argument is checked before anything is launched; a failed
 * check returns RET_ERR_INVALID_ARG (bad pointer, size, alignment or value)
 * or RET_ERR_UNSUPPORTED (a valid combination no kernel implements) and
 * launches nothing.  A failed launch returns RET_ERR_CUDA.  Kernels that wait
 * on an mbarrier give up after a bounded number of polls, set a device-side
 * error word and return; ret_check_device_error() reads it (RET_ERR_TIMEOUT).
 * No entry point aborts, traps or prints.  ret_last_error_string() describes
 * the last failure of the calling thread.
 */
#ifndef RETENTION_B200_H_
#define RETENTION_B200_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RET_OK = 0,
    RET_ERR_INVALID_ARG = 1,
    RET_ERR_UNSUPPORTED = 2,
    RET_ERR_CUDA = 3,
    RET_ERR_TIMEOUT = 4
} ret_status;

typedef enum { RET_F32 = 0, RET_BF16 = 1 } ret_dtype;

/*
 * xPos / rotary rotation of x [B, N, H, d], in place.
 * "Hybrid Architectures ...", sections 6.6 and 6.8: pair (2p, 2p+1) of the
 * vector at position n = pos_offset + t is turned by the angle n * theta_p,
 *     [x0', x1'] = [x0 cos - x1 sin, x0 sin + x1 cos],
 *     theta_p = theta_base^(-2p/d).
 * Queries and keys are both turned this way; their dot product then depends
 * only on the position difference (section 6.7).
 * x: device, dtype dt, 4-byte aligned.  d even, all sizes >= 1, theta_base > 0.
 */
ret_status ret_xpos_rotate(void* x, ret_dtype dt, int B, int N, int H, int d,
                           int64_t pos_offset, double theta_base, cudaStream_t stream);

/*
 * Chunkwise recurrent retention forward.
 * "Hybrid Architectures ...", section 7.2, and the RetNet paper summary,
 * Eq. 7: per chunk [i] of `chunk` tokens,
 *     out_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + (Q_[i] R_{i-1}) (.) xi,
 *     R_i     = gamma^chunk R_{i-1} + K_[i]^T (V_[i] (.) zeta),
 * xi_j = gamma^(j+1), zeta_j = gamma^(chunk-1-j) (0-based row j), R_0 = 0.
 * A last chunk of L < chunk tokens uses L in place of chunk.
 * q, k, v: device, dtype in_dt, 16-byte aligned, layouts above.
 * out: device [B, N, H, dv], dtype out_dt, 16-byte aligned; must not overlap
 *      q, k or v.
 * final_state: device fp32 [B, H, dk, dv] receiving R after the last token,
 *      or NULL.
 * xpos != 0 applies the rotation of ret_xpos_rotate (positions pos_offset + n,
 *      base theta_base) to q and k as they are loaded; the inputs are not
 *      modified.
 * Kernels: in_dt RET_BF16 with chunk 128, dk 128 or 256 and dv a multiple
 * of 64 (and dk 64 with chunk 64 or 128, zero-padded to 128 and computed in
 * 128-token blocks) runs on the tensor cores (tcgen05/TMEM/TMA) in two
 * launches: a pass that rotates q and k, scales the keys by the folded decay
 * and computes each head's masked intra-chunk scores once, then the kernel
 * of the read-out, P V and the state update.  Their scratch comes from a
 * stream-ordered memory pool the library keeps per device (allocated and
 * freed in stream order on `stream`; the pool keeps its memory for later
 * calls).  Heads whose decay is too fast for the folded factors
 * (gamma_h^64 < 2^-100) are computed by the token-by-token recurrent kernel
 * in the same call.  Other shapes: the fp32 CUDA-core chunkwise kernel when
 * its per-block working set (about 4 * chunk * (2 dk + chunk + 64)
 * + 256 dk bytes) fits in shared memory, else the recurrent kernel
 * (dk <= 256), which computes the same function.  Larger dk on neither path:
 * RET_ERR_UNSUPPORTED.  A failure to get scratch from the pool is
 * RET_ERR_CUDA; ret_forward_chunkwise_ws and ret_forward_chunkwise_noalloc
 * take none.
 */
ret_status ret_forward_chunkwise(const void* q, const void* k, const void* v,
                                 const double* gammas, int B, int N, int H, int dk, int dv,
                                 int chunk, void* out, float* final_state, cudaStream_t stream,
                                 ret_dtype in_dt, ret_dtype out_dt, int xpos,
                                 int64_t pos_offset, double theta_base);

/*
 * Chunkwise forward with a caller-provided device workspace: the same
 * computation and arguments as ret_forward_chunkwise, plus `workspace`
 * (device, 256-byte aligned, not overlapping any other buffer) of at least
 * ret_chunkwise_workspace_bytes(...) bytes.  The first launch writes into
 * it the rotated queries (when xpos != 0, or dk padded), the rotated keys
 * scaled by gamma^(a-j) (the decay of section 7.2 folded into the keys about
 * an anchor row a of each chunk: a = 127, or 63 for heads with
 * gamma^128 < 2^-60) and the masked scores P = tril(Q K'^T) of every
 * (batch, head, chunk) in bf16; the tensor-core kernel that follows reads
 * them by TMA.  Its contents are scratch and undefined after the call.  When
 * the shape does not take this path (ret_chunkwise_workspace_bytes returns
 * 0) or no head does (every gamma_h^64 < 2^-100), the call behaves as
 * ret_forward_chunkwise and does not touch the workspace; heads with
 * gamma_h^64 < 2^-100 among others are computed token by token beside it.
 * The path takes bf16 inputs with chunk 128, dk 128 or 256 and dv a multiple
 * of 64; dk = 64 with chunk 64 or 128 also runs on it, zero-padded to dk 128
 * in the workspace and blocked by 128 tokens (the result is the
 * recurrence's for any block length; states keep 64 rows).
 */
size_t ret_chunkwise_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk, ret_dtype in_dt,
                                     int xpos);

ret_status ret_forward_chunkwise_ws(const void* q, const void* k, const void* v,
                                    const double* gammas, int B, int N, int H, int dk, int dv,
                                    int chunk, void* out, float* final_state, cudaStream_t stream,
                                    ret_dtype in_dt, ret_dtype out_dt, int xpos,
                                    int64_t pos_offset, double theta_base, void* workspace,
                                    size_t workspace_bytes);

/*
 * The two launches of ret_forward_chunkwise_ws as separate calls, on the
 * same workspace, in stream order (prepare, then prepared).  Shapes outside
 * the workspace path (ret_chunkwise_workspace_bytes returns 0, or some head
 * with gamma_h^64 < 2^-100) return RET_ERR_UNSUPPORTED from both; use
 * ret_forward_chunkwise for them.
 *
 * ret_chunkwise_prepare reads q and k (device [B, N, H, dk], bf16, 16-byte
 * aligned) and fills the workspace with the rotated queries (xpos != 0), the
 * rotated, decay-scaled keys and the masked scores P of every chunk.  Its
 * arguments mean what they mean for ret_forward_chunkwise_ws; dv only
 * selects the path (a multiple of 64).
 *
 * ret_forward_chunkwise_prepared runs the tensor-core kernel on a workspace
 * that ret_chunkwise_prepare filled with the same q, k, gammas, B, N, H, dk,
 * chunk, xpos, pos_offset and theta_base (the workspace is only read).  It
 * can continue a sequence: initial_state (device fp32 [B, H, dk, dv], 16-byte
 * aligned, or NULL for the zero state) is the state S after every token
 * before this call's first one, and the call computes
 *     S_n = gamma_h S_{n-1} + k_n v_n^T from S = initial_state,  o_n = q_n^T S_n,
 * i.e. the chunkwise recurrence with R_0 = initial_state ("Hybrid
 * Architectures: RetNet and the Three Computation Paradigms", section 7.2;
 * RetNet paper summary, chunkwise representation, Eq. 7, and inference
 * protocol).  With pos_offset set to the number of earlier tokens, splitting
 * a sequence into calls that pass each call's final_state on as the next
 * call's initial_state gives the single call's outputs and final state up
 * to rounding.  final_state may be the same buffer as initial_state (updated
 * in place); any other overlap is RET_ERR_INVALID_ARG.
 */
/* Workspace bytes of ret_chunkwise_prepare / ret_forward_chunkwise_prepared
 * (0 when the shape is outside the path): the rotated queries (xpos, or a
 * dk of 64 padded to 128) and the rotated, decay-scaled keys, [B, N, H, dk]
 * bf16 each at the kernel's dk, then (256-byte aligned) the P tiles,
 * [B, H, ceil(N / 128), 128, 128] bf16.  The same as
 * ret_chunkwise_workspace_bytes. */
size_t ret_chunkwise_prepare_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk,
                                             ret_dtype in_dt, int xpos);

ret_status ret_chunkwise_prepare(const void* q, const void* k, const double* gammas, int B, int N,
                                 int H, int dk, int dv, int chunk, cudaStream_t stream,
                                 ret_dtype in_dt, int xpos, int64_t pos_offset, double theta_base,
                                 void* workspace, size_t workspace_bytes);

ret_status ret_forward_chunkwise_prepared(const void* q, const void* k, const void* v,
                                          const double* gammas, int B, int N, int H, int dk,
                                          int dv, int chunk, void* out, float* final_state,
                                          const float* initial_state, cudaStream_t stream,
                                          ret_dtype in_dt, ret_dtype out_dt, int xpos,
                                          int64_t pos_offset, double theta_base,
                                          const void* workspace, size_t workspace_bytes);

/*
 * Gradients of the chunkwise forward: given dout = dL/d(out), the gradients
 * of L with respect to q, k and v of ret_forward_chunkwise (same q, k, v,
 * gammas, sizes, xpos, pos_offset, theta_base).  They are the derivatives of
 * the definition o_n = sum_{m<=n} gamma^(n-m) (q'_n . k'_m) v_m ("Hybrid
 * Architectures ...", section 2.1; RetNet paper summary, Eq. 6), with
 * q' = R q and k' = R k the rotated vectors (section 6.8; identity when
 * xpos = 0):
 *     dq = R^T sum_{m<=n} gamma^(n-m) (dout_n . v_m) k'_m
 *     dk = R^T sum_{n>=m} gamma^(n-m) (dout_n . v_m) q'_n
 *     dv =     sum_{n>=m} gamma^(n-m) (q'_n . k'_m)  dout_n
 * The pages train through the chunkwise form but print no backward pass;
 * these are its plain derivatives.  Each sum is computed as a tensor-core
 * chunkwise retention pass (the two anti-causal ones on the time-reversed
 * sequence), so the same path constraints apply: bf16 q, k, v, dout
 * (device [B, N, H, d], 16-byte aligned), chunk = 128, dk 128 or 256, dv a
 * multiple of 128 and every gamma_h^128 >= 2^-60, else RET_ERR_UNSUPPORTED.
 * dq, dk: device fp32 [B, N, H, dk]; dv: device fp32 [B, N, H, dv]; written,
 * 16-byte aligned, overlapping nothing else.
 * workspace: device, 256-byte aligned, at least
 * ret_backward_workspace_bytes(...) bytes (the rotated keys in both time
 * orders, the rotated queries, v and dout time-reversed, all bf16, and the
 * scratch of two concurrent passes), overlapping nothing else.
 * Half of the passes run on a second CUDA stream that the library creates
 * per device on first use and keeps for the life of the process; the call
 * joins it back into `stream` with events before returning (also under
 * CUDA-graph capture).
 */
size_t ret_backward_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk, ret_dtype in_dt,
                                    int xpos);

ret_status ret_backward_chunkwise(const void* q, const void* k, const void* v, const void* dout,
                                  const double* gammas, int B, int N, int H, int dk, int dv,
                                  int chunk, float* dq, float* dk_out, float* dv_out,
                                  cudaStream_t stream, ret_dtype in_dt, int xpos,
                                  int64_t pos_offset, double theta_base, void* workspace,
                                  size_t workspace_bytes);

/*
 * Retention with the score normalizations 2 and 3 ("Hybrid Architectures
 * ...", section 8.5; RetNet paper summary, "Retention Score
 * Normalization"), selected by norm_flags:
 *   RET_NORM_DECAY  the decay matrix row-normalized,
 *                   D~_nm = D_nm / sqrt(sum_{i<=n} D_ni);
 *   RET_NORM_SCORE  the scores row-normalized,
 *                   R~_nm = R_nm / max(|sum_{i<=n} R_ni|, 1),
 *                   R = (Q K^T) (.) D~ (or D without RET_NORM_DECAY);
 * out = R~ V.  Normalization 1 (the 1/sqrt(d) on Q K^T) is the caller's
 * scaling of q.  The row sums run over the whole sequence: position pos_offset
 * + n is row pos_offset + n of D, and the score row sum is q_n . z_n with
 * z_n = gamma_h z_{n-1} + k_n, the decayed key sum (rotated keys with xpos).
 * Both normalizations multiply output row n by a positive scalar and leave
 * the state S unchanged.  The pages take the absolute value of the sum (not
 * the sum of absolute values); so does this library, which keeps the
 * chunkwise and recurrent forms exact.
 */
#define RET_NORM_DECAY 1
#define RET_NORM_SCORE 2

/*
 * Chunkwise forward with the normalizations: arguments as
 * ret_forward_chunkwise_prepared (same path constraints: bf16 inputs, chunk
 * 128, dk 128 or 256, dv a multiple of 64, every gamma_h^128 >= 2^-60, else
 * RET_ERR_UNSUPPORTED), plus
 *   norm_flags  a combination of RET_NORM_DECAY and RET_NORM_SCORE (0: the
 *               plain retention);
 *   initial_z   device fp32 [B, H, dk], 16-byte aligned, or NULL (zero): z
 *               after every token before this call's first one;
 *   final_z     device fp32 [B, H, dk], 16-byte aligned, or NULL: z after
 *               the last token (may be the same buffer as initial_z);
 *   workspace   device, 256-byte aligned, at least
 *               ret_normalized_workspace_bytes(...) bytes, scratch.
 * Splitting a sequence into calls that hand final_state and final_z on, with
 * pos_offset the number of earlier tokens, gives the single call's result.
 * No buffer may overlap another except final_state = initial_state and
 * final_z = initial_z.
 */
size_t ret_normalized_workspace_bytes(int B, int N, int H, int dk, int dv, int chunk,
                                      ret_dtype in_dt, int xpos);

ret_status ret_forward_chunkwise_normalized(const void* q, const void* k, const void* v,
                                            const double* gammas, int B, int N, int H, int dk,
                                            int dv, int chunk, int norm_flags, void* out,
                                            const float* initial_state, float* final_state,
                                            const float* initial_z, float* final_z,
                                            cudaStream_t stream, ret_dtype in_dt,
                                            ret_dtype out_dt, int xpos, int64_t pos_offset,
                                            double theta_base, void* workspace,
                                            size_t workspace_bytes);

/*
 * One decode step with the normalizations: as ret_decode_step, then the
 * output multiplied by c / max(|c q.z|, 1) (RET_NORM_SCORE; c = 1 without
 * RET_NORM_DECAY), c = 1 / sqrt(sum_{i<=position} gamma_h^i), after
 * z <- gamma_h z + k.  position: the token's 0-based position in its
 * sequence, >= 0.  z: device fp32 [B, H, dk], 16-byte aligned, updated in
 * place; required with RET_NORM_SCORE, ignored (may be NULL) without.
 */
ret_status ret_decode_step_normalized(const void* q, const void* k, const void* v,
                                      const double* gammas, float* state, float* z, void* out,
                                      int64_t position, int norm_flags, cudaStream_t stream,
                                      int B, int H, int dk, int dv, ret_dtype in_dt,
                                      ret_dtype out_dt);

/*
 * One decode step for a batch of sequences that sit at different positions
 * (serving: "Hybrid Architectures ...", section 5.2; RetNet paper summary,
 * inference protocol).  positions: device int64 [B], 8-byte aligned, the
 * 0-based position of this token in sequence b (>= 0; not read back on the
 * host).  With xpos != 0, q and k of sequence b are turned by the xPos
 * rotation at positions[b] (section 6.8, theta_base as in ret_xpos_rotate;
 * dk even) inside the step.  norm_flags and z as in
 * ret_decode_step_normalized, at each sequence's own position (0: none,
 * z may be NULL).  Otherwise as ret_decode_step.
 */
ret_status ret_decode_step_positions(const void* q, const void* k, const void* v,
                                     const double* gammas, float* state, float* z, void* out,
                                     const int64_t* positions, int xpos, double theta_base,
                                     int norm_flags, cudaStream_t stream, int B, int H, int dk,
                                     int dv, ret_dtype in_dt, ret_dtype out_dt);

/*
 * Allocation-free variant of ret_forward_chunkwise_ws, for callers that
 * cannot allocate device memory at call time: for example a plug-in that runs
 * inside a host framework which owns all device memory and hands out no
 * allocator, or a service that fixes its memory footprint at start-up and
 * forbids allocation afterwards.  The pages have no counterpart; this is a
 * deployment convenience of this library.
 * Same arguments and results as ret_forward_chunkwise (the caller still
 * passes every input and output buffer).  It runs the two-pass form (the
 * rotation / key-scaling pass, then the tensor-core kernel computing the
 * masked scores itself, so no P tiles), whose scratch is a fixed device
 * array inside the library, of
 * ret_chunkwise_noalloc_max_bytes() bytes (64 MiB) on every GPU that loads
 * the library, held until the process exits.  Problems needing more scratch
 * than that return RET_ERR_INVALID_ARG, shapes outside the workspace path
 * RET_ERR_UNSUPPORTED; nothing is allocated in either case.  The scratch is
 * B*N*H*dk*4 bytes with xpos and B*N*H*dk*2 without, for dk 128 or 256;
 * for dk = 64 (padded to 128 inside, the queries always copied) it is
 * B*N*H*128*4 bytes with or without xpos.
 * The first call on a device looks up the array's device address (once per
 * device and CUDA context, with that device current); make that first call
 * before any stream capture.  After a cudaDeviceReset the next call looks
 * the address up again in the new context.  All calls share the one array
 * and leave their scratch in it;
 * nothing in it needs to start at zero.  Calls whose kernels overlap on the
 * GPU (other streams, other host threads) race on the array: serialise them.
 */
ret_status ret_forward_chunkwise_noalloc(const void* q, const void* k, const void* v,
                                         const double* gammas, int B, int N, int H, int dk, int dv,
                                         int chunk, void* out, float* final_state,
                                         cudaStream_t stream, ret_dtype in_dt, ret_dtype out_dt,
                                         int xpos, int64_t pos_offset, double theta_base);

/* Size in bytes of the fixed scratch array of ret_forward_chunkwise_noalloc. */
size_t ret_chunkwise_noalloc_max_bytes(void);

/*
 * One recurrent decode step, state updated in place.
 * "Hybrid Architectures ...", sections 2.1 and 5.2; RetNet paper summary,
 * recurrent representation and inference protocol:
 *     S <- gamma_h S + k v^T,   out = q^T S   (read-out after the update).
 * q, k: device [B, H, dk], v: device [B, H, dv], dtype in_dt.
 * state: device fp32 [B, H, dk, dv], read and written in place, 16-byte
 *        aligned, dv a multiple of 4.
 * out: device [B, H, dv], dtype out_dt.
 */
ret_status ret_decode_step(const void* q, const void* k, const void* v, const double* gammas,
                           float* state, void* out, cudaStream_t stream, int B, int H, int dk,
                           int dv, ret_dtype in_dt, ret_dtype out_dt);

/*
 * Parallel form, O(N^2), for cross-checking the chunkwise path on the GPU.
 * "Hybrid Architectures ...", sections 4.2-4.3; RetNet paper summary, Eq. 5:
 *     out = (Q K^T (.) D) V,  D_nm = gamma^(n-m) for n >= m, else 0.
 * Arguments as ret_forward_chunkwise (no chunk, no state).  fp32 arithmetic
 * on the CUDA cores.  dk <= 256.
 */
ret_status ret_forward_parallel(const void* q, const void* k, const void* v,
                                const double* gammas, int B, int N, int H, int dk, int dv,
                                void* out, cudaStream_t stream, ret_dtype in_dt, ret_dtype out_dt,
                                int xpos, int64_t pos_offset, double theta_base);

/*
 * Recurrent form over a whole sequence, token by token, for cross-checking
 * the chunkwise path on the GPU ("Hybrid Architectures ...", section 2.1).
 * Arguments as ret_forward_chunkwise (no chunk).  The state lives in
 * registers in fp32.  dk <= 256.
 */
ret_status ret_forward_recurrent(const void* q, const void* k, const void* v,
                                 const double* gammas, int B, int N, int H, int dk, int dv,
                                 void* out, float* final_state, cudaStream_t stream,
                                 ret_dtype in_dt, ret_dtype out_dt, int xpos,
                                 int64_t pos_offset, double theta_base);

/*
 * MultiScaleRetention layer forward ("Hybrid Architectures ...", section 9.1;
 * RetNet paper summary, "Gated Multi-Scale Retention"):
 *     Q = rot(X W_Q), K = rot(k_scale X W_K), V = X W_V, G = X W_G,
 *     Y_h = Retention(Q_h, K_h, V_h; gamma_h)          (chunkwise, `chunk`)
 *     Z = swish(G) (.) GroupNorm_H(Y),  out = Z W_O,
 * GroupNorm per (token, head) over the head's d_v channels with biased
 * variance, eps inside the square root and no affine term; swish(x) =
 * x sigmoid(x).
 * X [B, N, d_model] bf16; W_Q, W_K [d_model, H dk], W_V, W_G [d_model, H dv],
 * W_O [H dv, d_model], all bf16 row-major as (input, output); out
 * [B, N, d_model] of dtype out_dt.  All device, 16-byte aligned.
 * workspace: device, 256-byte aligned, at least ret_msr_workspace_bytes(...)
 * bytes, overlapping nothing; scratch, undefined after the call.
 * xpos/pos_offset/theta_base as in ret_forward_chunkwise.  Requires chunk
 * 128, dk 128 or 256, dv in {128, 256, 512, 1024}, d_model a multiple of 8
 * and every gamma_h^128 >= 2^-60 (else RET_ERR_UNSUPPORTED).
 * Five launches on `stream`: the (cos, sin) table of the rotation (xpos), the
 * projections (tcgen05 GEMM with the rotation, k_scale, the chunkwise key
 * decay and swish fused in its epilogue), the chunkwise retention, GroupNorm
 * with the gate, and the output projection.
 */
size_t ret_msr_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv);

ret_status ret_msr_forward(const void* X, const void* Wq, const void* Wk, const void* Wv,
                           const void* Wg, const void* Wo, const double* gammas, int B, int N,
                           int dmodel, int H, int dk, int dv, int chunk, double k_scale, double eps,
                           int xpos, int64_t pos_offset, double theta_base, void* out,
                           ret_dtype out_dt, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/*
 * One RetNet block, pre-LayerNorm residual layout ("Hybrid Architectures
 * ...", section 9.2; RetNet paper summary, "Overall RetNet Architecture"):
 *     Y   = MSR(LN1(X)) + X
 *     out = gelu(LN2(Y) W1) W2 + Y
 * MSR as ret_msr_forward (same weights, shapes, k_scale, gn_eps, xpos and
 * path constraints); LN(x) = (x - mean) / sqrt(var + ln_eps) * gain + bias
 * per token over d_model (biased variance); gelu(x) = x Phi(x) with the exact
 * normal CDF.  The pages' RetNet uses d_ff = 2 d_model.
 * X [B, N, d_model] bf16; W1 [d_model, d_ff], W2 [d_ff, d_model] bf16
 * row-major as (input, output); ln*_gain, ln*_bias: bf16 [d_model], or NULL
 * (gain 1, bias 0); out [B, N, d_model] of dtype out_dt.  Y, the LayerNorm
 * outputs and the FFN hidden layer are held in bf16 in the workspace
 * (device, 256-byte aligned, at least ret_retnet_block_workspace_bytes(...)
 * bytes, overlapping nothing).  d_model and d_ff multiples of 8.
 * Eight launches: LayerNorm, the MSR's five (the residual added in the output
 * projection's epilogue), LayerNorm, and the two FFN GEMMs (gelu and the
 * residual in their epilogues).
 */
size_t ret_retnet_block_workspace_bytes(int B, int N, int dmodel, int H, int dk, int dv, int dff);

ret_status ret_retnet_block_forward(const void* X, const void* ln1_gain, const void* ln1_bias,
                                    const void* Wq, const void* Wk, const void* Wv, const void* Wg,
                                    const void* Wo, const void* ln2_gain, const void* ln2_bias,
                                    const void* W1, const void* W2, const double* gammas, int B,
                                    int N, int dmodel, int H, int dk, int dv, int dff, int chunk,
                                    double k_scale, double gn_eps, double ln_eps, int xpos,
                                    int64_t pos_offset, double theta_base, void* out,
                                    ret_dtype out_dt, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream);

/*
 * Y = X W on the tensor cores (the GEMM of the MSR layer): X [M, K] bf16,
 * W [K, N] bf16, row-major; Y [M, N] of dtype out_dt.  fp32 accumulation.
 * N and K multiples of 8; device pointers 16-byte aligned; Y must not overlap
 * X or W.
 */
ret_status ret_linear_bf16(const void* X, const void* W, void* Y, int M, int N, int K, ret_dtype out_dt,
                           cudaStream_t stream);

/*
 * Diagnostics: one device thread waits on a barrier that nothing arrives on,
 * with the same bounded wait as the tensor-core kernels, for `polls` polls
 * (1 .. 2^24), gives up and sets the device error word.  The following
 * ret_check_device_error on the stream returns RET_ERR_TIMEOUT (and clears
 * the word); the context stays usable.  It exercises the timeout path
 * without hanging or faulting the GPU.
 */
ret_status ret_selftest_bounded_wait(uint32_t polls, cudaStream_t stream);

/*
 * Synchronises `stream`, then reports (and clears) the device-side error word
 * that kernels set when a bounded wait gives up.  RET_OK if none was set.
 */
ret_status ret_check_device_error(cudaStream_t stream);

/* Description of the calling thread's last failure ("" if none). */
const char* ret_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* RETENTION_B200_H_ */
