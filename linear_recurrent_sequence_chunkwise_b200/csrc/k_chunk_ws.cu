// k_chunk_ws.cu -- chunkwise retention forward on the tensor cores: a
// warp-specialized tcgen05 / TMEM / TMA kernel, fed either by a
// bandwidth-bound rotation pass (two-pass form) or by its own CTAs (fused
// form).
//
// Mathematics ("Hybrid Architectures: RetNet and the Three Computation
// Paradigms", section 7.2; RetNet paper summary, Eq. 7).  For a chunk of L
// rows and 0-based rows r, c:
//     out_r = sum_{c<=r} gamma^(r-c) (q_r . k_c) v_c + gamma^(r+1) q_r^T R_prev
//     R     = gamma^L R_prev + sum_c gamma^(L-1-c) k_c v_c^T
// The kernel folds every decay factor into one scaled key and one row scale
// about an anchor row a (a = min(anchor_h, L-1), anchor_h 127 or 63):
//     k'_c  = gamma^(a-c) k_c
//     T     = gamma^(a+1) R_prev                      (read-out copy, bf16)
//     out_r = gamma^(r-a) [ sum_{c<=r} (q_r . k'_c) v_c + q_r^T T ]
//     R     = gamma^L R_prev + gamma^(L-1-a) K'^T V
// since gamma^(r-c) = gamma^(r-a) gamma^(a-c) and gamma^(r+1) = gamma^(r-a)
// gamma^(a+1).  So the decay mask D becomes a plain causal mask on Q K'^T,
// generated in registers, and the intra-chunk scores, the cross read-out and
// the state update each feed one fp32 TMEM accumulator.  With a = L-1 (heads
// with gamma^128 >= 2^-60) the factors are those of the pages' zeta and xi;
// faster-decaying heads take a = 63, which keeps every factor within
// 2^+-100 for gamma^64 >= 2^-100; heads below that are left to the recurrent
// kernel (their CTAs return at once).
//
// 1. k_prep_qk (HBM-bound, one pass, two-pass form): rotates q and k once per
//    head (xPos, consecutive pairs, angle (pos_offset + n) theta_p with the
//    sine and cosine of each (position, pair) evaluated once for all heads),
//    scales each rotated key row by gamma^(a-c), and writes q_rot and k'
//    (bf16) into the workspace.  Without rotation only k' is written and q is
//    read in place.
// 2. k_chunkwise_ws: one CTA per (batch, head, 64 value columns), 16 warps
//    in five roles (registers rebalanced with setmaxnreg):
//      warp 0  TMA producer: L2 prefetch two chunks ahead (the CTAs of a
//              head split the boxes), then per chunk the Q tile into a
//              staging buffer, the K' tile in parts of 128 d_k rows through
//              a 3-slot ring, and the V tile (2 slots);
//      warp 1  tensor pipe, first issuer (one elected lane), per chunk j
//                A  = Q K'^T          (Q from TMEM, K' from smem), part by part,
//                O  = Q T             (read-out of the state before chunk j),
//                O += P V             (P from TMEM; each operand behind its
//                                      own barrier, V's TMA barrier included);
//      warp 3  tensor pipe, second issuer: the state update dS = K'^T V of
//              each K' part, beside warp 1's stream (each K' slot is free
//              once both issuers have read it);
//      warp 2  output store: one TMA store (or reduce-add) of each staged
//              output tile;
//      warps 4-7 (Q warpgroup): the staged Q of chunk j+1 -> registers as
//                soon as it lands, -> TMEM once the read-out of chunk j is
//                done; a plain smem read keeps the load traffic on the TMA
//                path (per-row global loads from these threads measurably
//                slow the tensor pipe down).  In the fused form these warps
//                also rotate this CTA's share of each chunk into the head's
//                exchange ring (see q_role_fused);
//      warps 8-15 (two warpgroups on TMEM lanes 0..127, one column half each):
//                mask:     P = tril(A) -> packed bf16 in TMEM,
//                state:    R = gamma^L R + gamma^(L-1-a) dS in registers
//                          (fp32), then the bf16 T = gamma^(a'+1) R into smem
//                          for the next read-out,
//                epilogue: out = gamma^(r-a) O staged in the chunk's V slot.
//    TMEM columns: A [0,128), P [128,192), O [192,256), Q [256,384),
//    dS [384,512).  Every hand-off between the roles has at least one block
//    of MMAs in between, so no role waits on another in the steady state.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "kernels.h"
#include "tc_util.cuh"
#include "tmap.h"

namespace ret {

static __device__ int g_err_chunk_ws = 0;

cudaError_t read_clear_error_chunk_ws(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_err_chunk_ws, sizeof(int));
    if (e == cudaSuccess && *flag) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_err_chunk_ws, &zero, sizeof(int));
    }
    return e;
}

namespace {

constexpr int kC = 128;           // chunk rows (M of every MMA)
constexpr int kW = 64;            // d_v columns per CTA
constexpr int kPartDk = 128;      // d_k rows per pipeline part (one state block)
constexpr int kVBytes = kC * kW * 2;              // 16 KB
constexpr int kThreads = 512;   // control warpgroup (TMA, MMA), Q warpgroup, two transform warpgroups

// ------------------------------------------------------------------ prep

// One warp per (batch, token); lanes walk groups of 8 d_k elements (4 pairs).
// Rows have dkr elements in memory (dkr <= DK); groups past dkr are written
// as zeros (a smaller d_k padded to the kernel's).  With qcopy the queries
// are written to q_rot, turned only with xpos.
template <int DK>
__global__ void __launch_bounds__(256) k_prep_qk(const __nv_bfloat16* __restrict__ q,
                                                  const __nv_bfloat16* __restrict__ k,
                                                  __nv_bfloat16* __restrict__ q_rot,
                                                  __nv_bfloat16* __restrict__ k_out, HeadConsts hc, int B, int N,
                                                  int H, int chunk, int xpos, long long pos0, double log2base,
                                                  int q_ld, int k_ld, int dkr, int qcopy) {
    // theta_p = base^(-2p/dkr), once per block (fp64, as the rotation's reference)
    __shared__ double s_theta[DK / 2];
    for (int i = threadIdx.x; i < DK / 2; i += blockDim.x) s_theta[i] = exp2(-2.0 * i / dkr * log2base);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const long long t = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // b * N + n
    if (t >= (long long)B * N) return;
    const int n = (int)(t % N);
    const int r = n % chunk;
    const int L = min(chunk, N - (n - r));
    constexpr int kGroups = DK / 8;
    for (int g = lane; g < kGroups; g += 32) {
        if (8 * g >= dkr) {  // padding
            for (int hh = 0; hh < H; hh++) {
                const size_t e = ((size_t)t * H + hh) * DK + 8 * g;
                *reinterpret_cast<uint4*>(k_out + e) = make_uint4(0, 0, 0, 0);
                if (qcopy) *reinterpret_cast<uint4*>(q_rot + e) = make_uint4(0, 0, 0, 0);
            }
            continue;
        }
        float cs[4], sn[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            cs[i] = 1.f;
            sn[i] = 0.f;
            if (xpos) sincosf(rot_angle(pos0 + n, s_theta[4 * g + i]), &sn[i], &cs[i]);
        }
        // The loads of kHB heads are issued together (memory-level
        // parallelism), then rotated and stored.
        constexpr int kHB = 8;
        for (int h0 = 0; h0 < H; h0 += kHB) {
            uint4 kw[kHB], qw[kHB];
#pragma unroll
            for (int hh = 0; hh < kHB; hh++) {
                if (h0 + hh < H) {
                    const size_t row = (size_t)t * H + h0 + hh;
                    kw[hh] = __ldg(reinterpret_cast<const uint4*>(k + row * k_ld + 8 * g));
                    if (qcopy) qw[hh] = __ldg(reinterpret_cast<const uint4*>(q + row * q_ld + 8 * g));
                }
            }
#pragma unroll
            for (int hh = 0; hh < kHB; hh++) {
                if (h0 + hh >= H) continue;
                const size_t e = ((size_t)t * H + h0 + hh) * DK + 8 * g;
                // k' scale gamma^(a-r), a = min(anchor, L-1): the exponent in fp64,
                // exp2 in fp32 (relative error ~1e-7)
                const int a = min(hc.anchor[h0 + hh], L - 1);
                const float zeta = exp2f((float)((double)(a - r) * hc.log2g[h0 + hh]));
                uint32_t* kwv = reinterpret_cast<uint32_t*>(&kw[hh]);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const float x0 = tc::bf16lo(kwv[i]), x1 = tc::bf16hi(kwv[i]);
                    const float c = cs[i] * zeta, s = sn[i] * zeta;
                    kwv[i] = tc::pack_bf16x2(x0 * c - x1 * s, x0 * s + x1 * c);
                }
                *reinterpret_cast<uint4*>(k_out + e) = kw[hh];
                if (qcopy) {
                    uint32_t* qwv = reinterpret_cast<uint32_t*>(&qw[hh]);
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const float x0 = tc::bf16lo(qwv[i]), x1 = tc::bf16hi(qwv[i]);
                        qwv[i] = tc::pack_bf16x2(x0 * cs[i] - x1 * sn[i], x0 * sn[i] + x1 * cs[i]);
                    }
                    *reinterpret_cast<uint4*>(q_rot + e) = qw[hh];
                }
            }
        }
    }
}

// ------------------------------------------------------------- main kernel

struct WsParams {
    CUtensorMap tq, tk, tv;
    CUtensorMap to;       // out, stored by TMA from the staged tile (tma_out); fp32 in two column halves
    int tma_out;
    void* out;
    float* fstate;
    const float* istate;  // state before the first token, [B, H, DK, dv] fp32, or null (zero)
    int N, H, dv;
    int accumulate;       // fp32 out only: out += result
    int out_rev;          // output of token n goes to row N-1-n
    int dks;              // rows of the states (d_k before padding)
    const float* rowscale;  // [B, N, H] factor of each output row, or null
    int nmain;            // CTAs: B * H * (dv / 64), one per (b, h, 64 value columns)
    HeadConsts hc;
    // Fused rotation (FUSED instances).  A launch takes the (b, h) pairs
    // bh0 .. bh0 + gridDim.x / nt - 1 (nt = dv / 64 CTAs per head; bh0 = 0
    // otherwise).  Each of a head's nt CTAs turns its 1/nt share of the rows
    // of every chunk (xPos) from the raw q and k, scales the keys by zeta,
    // and writes them into the head's exchange ring (kRing chunk slots in
    // global memory, small enough to stay in L2); the tensor maps tq / tk
    // then point at the ring.  Per (head g, slot) two counts: ready[g][slot]
    // the shares written into the slot, consumed[g][slot] the CTAs whose
    // loads of the slot's chunk have landed (which frees it).  Chunk i lives
    // in slot i % kRing as its generation u = i / kRing, so it is complete
    // when ready reaches nt (u + 1), and the slot may take chunk i + kRing
    // once consumed reaches nt (u + 1).  (The CTAs of a head drift apart by
    // up to kLead chunks, so one count per head would not say which chunk.)
    int bh0;
    const __nv_bfloat16* q_raw;
    const __nv_bfloat16* k_raw;
    int q_ld, k_ld;       // elements between consecutive (token, head) rows of q_raw / k_raw
    __nv_bfloat16* ring_q;
    __nv_bfloat16* ring_k;
    unsigned int* ready;
    unsigned int* consumed;
    int xpos;
    long long pos0;
    double log2base;
};

// Exchange ring of the fused rotation: chunk slots per head, and how many
// chunks ahead of the one being computed the shares are written.
constexpr int kRing = 6, kLead = 3;

// Wait (bounded) until *ctr >= target, with acquire semantics at GPU scope,
// then order the caller's later async-proxy (TMA) accesses after what it saw.
__device__ __forceinline__ bool wait_count(const unsigned int* ctr, unsigned int target) {
    for (uint32_t i = 0; i < (1u << 22); i++) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return true;
        }
        __nanosleep(32);
    }
    return false;
}

__device__ __forceinline__ void count_release(unsigned int* ctr) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

// Named barrier 1 over the Q warpgroup (warps 4-7): returns whether x holds
// in all 128 threads; also orders their memory accesses around it.
__device__ __forceinline__ bool qwg_all(bool x) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)x)
        : "memory");
    return r != 0;
}

constexpr int kKSlots = 3;                         // K' ring depth (parts of 128 d_k rows)
constexpr int kKPartBytes = kPartDk * kC * 2;      // 32 KB

template <int DK>
struct WsSmem {
    static constexpr uint32_t kQ = 0;                              // Q staging, DK x 128 rows
    static constexpr uint32_t kK = kQ + DK * kC * 2;               // K' ring
    static constexpr uint32_t kV = kK + kKSlots * kKPartBytes;     // 2 x 16 KB
    static constexpr uint32_t kT = kV + 2 * kVBytes;               // DK x 128 B
    static constexpr uint32_t kEnd = kT + DK * 128;
    static constexpr uint32_t kBytes = kEnd + 1024;
};

// TMEM columns: A = Q K'^T (fp32), P (packed bf16), O (fp32), Q (packed
// bf16, the A operand of Q K'^T and of the read-out), dS = K'^T V (fp32).
constexpr uint32_t kTA = 0, kTP = 128, kTO = 192, kTQ = 256, kTD = 384;

// Per-thread register budgets of the three warpgroup roles.  The block is
// launched with 512 threads x 128 registers (ptxas reports 128 for every
// instance); the budgets add up to 128 * (72 + 136) + 256 * 152 = 65536.
constexpr int kRegsCtl = 72, kRegsQ = 136, kRegsXf = 152;
static_assert(128 * (kRegsCtl + kRegsQ) + 256 * kRegsXf <= 512 * 128, "register split exceeds the launch allocation");

struct Bars {
    uint64_t qfull, qempty, kfull[kKSlots], kempty[kKSlots], vfull[2], vempty[2];
    uint64_t qready, qtm, afull, aread, pready, dsdone, dsfree, tready, ofull, ofree, ostaged[2], ostaged2[2], ohalf[2];
};

__device__ __forceinline__ void elect_arrive(uint64_t* bar, int lane) {
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(bar);
}

template <int N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// An angle (fp64) reduced to [-pi, pi] and rounded to fp32, for the fast
// fp32 sine and cosine (absolute error a few 1e-7 there).
__device__ __forceinline__ float angle_mod_2pi(double a) {
    const double two_pi = 6.283185307179586476925286766559, inv_two_pi = 0.15915494309189533576888376337251;
    return (float)fma(-two_pi, rint(a * inv_two_pi), a);
}

// One 16-byte group (4 consecutive pairs) of a row, turned by the angles
// whose cosines and sines are c[], s[] (k rows: already scaled by zeta).
__device__ __forceinline__ uint4 turn_group(uint4 x, const float (&c)[4], const float (&s)[4]) {
    uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float x0 = tc::bf16lo(w[i]), x1 = tc::bf16hi(w[i]);
        w[i] = tc::pack_bf16x2(x0 * c[i] - x1 * s[i], x0 * s[i] + x1 * c[i]);
    }
    return x;
}

// The Q warpgroup of the fused instances.  Per chunk jq:
//   * once the read-out of chunk jq - 1 has consumed the previous Q, the
//     staged Q goes from shared memory into TMEM one 64-column slab at a time
//     (few registers held), and the tensor pipe is told (qready);
//   * the count of the chunk written in the previous iteration is released
//     (its bulk stores have long completed, so this is cheap);
//   * this CTA's share of chunk jq + kLead is written into the exchange ring,
//     once the slot is free (every CTA of the head has loaded the chunk that
//     last used it: consumed[g][slot] = nt * generation; the count is read one
//     iteration early).  The share is the rows [r0, r0 + R) of the chunk,
//     R = ceil(128 / nt); each thread turns one 16-byte group (pairs
//     4g .. 4g+3) of every kStep-th row, writes it into the Q staging buffer
//     (free until the staging buffer is handed back), and one thread copies
//     the rows into the ring with bulk stores (pieces of up to 64 rows);
//   * the staging buffer goes back to the TMA producer (qempty), and the raw
//     rows of chunk jq + kLead + 1 are loaded into registers for the next
//     iteration (their latency is hidden).
// The rotation of a thread's first row is evaluated from the position (fp64
// angle, reduced, then fp32 sine and cosine), the next ones by turning it
// through kStep * theta_p; keys are also scaled by gamma^(a-r); rows past the
// end of the sequence and groups past the caller's d_k are written as zeros.
// The rows of the prologue (chunks 0 .. kLead - 1) are written before the
// loop, and the staging buffer is handed to the producer once (qempty phase
// 0) before it loads the first Q.  The warpgroup agrees on every wait's
// outcome (named barrier 1), so a timed-out wait cannot strand part of it at
// a barrier.  Returns false on a timeout.
template <int DK>
__device__ __forceinline__ bool q_role_fused(const WsParams& p, uint8_t* sQ, uint32_t tb, uint32_t lane_off, int r,
                                             int quarter, int lane, int nt, int jt, int gl, int b, int h,
                                             int nchunks, double lg, int anc, Bars& bars) {
    constexpr int kGpr = DK / 8;             // 16-byte groups in a row
    constexpr int kRpw = 32 / kGpr;          // rows one warp covers at a time
    constexpr int kStep = 4 * kRpw;          // rows between one thread's rows
    constexpr int kBatch = 4;                // rows whose loads are in flight together
    constexpr int kPiece = (DK * kC * 2) / (4 * DK);   // rows of q and k the staging buffer holds (64)
    const int N = p.N, H = p.H;
    const int grp = lane % kGpr;
    const int rsub = quarter * kRpw + lane / kGpr;     // row offset within a step
    const bool real = 8 * grp < p.dks;       // inside the caller's d_k
    const bool turn = p.xpos && real;
    const int wtid = quarter * 32 + lane;
    const int R = (kC + nt - 1) / nt;
    const int r0 = min(R * jt, kC), r1 = min(r0 + R, kC);
    // theta_p = base^(-2p/d_k) of the thread's four pairs (fp64), and the
    // turn through kStep positions
    double theta[4];
    float cstep[4], sstep[4];
    {
        const double inv_dk = 1.0 / p.dks;
#pragma unroll
        for (int k = 0; k < 4; k++) {
            theta[k] = turn ? exp2(-2.0 * (4 * grp + k) * inv_dk * p.log2base) : 0.0;
            cstep[k] = 1.f;
            sstep[k] = 0.f;
            if (turn) __sincosf(angle_mod_2pi((double)kStep * theta[k]), &sstep[k], &cstep[k]);
        }
    }
    auto raw_row = [&](int i, int rr) { return ((size_t)b * N + (size_t)i * kC + rr) * H + h; };
    // the raw rows rb, rb + kStep, ... (kBatch of them) of chunk i
    auto load_rows = [&](int i, int rb, uint4 (&qw)[kBatch], uint4 (&kw)[kBatch]) {
        const int L = i < nchunks ? min(kC, N - i * kC) : 0;
#pragma unroll
        for (int u = 0; u < kBatch; u++) {
            const int rr = rb + u * kStep;
            qw[u] = kw[u] = make_uint4(0, 0, 0, 0);
            if (real && rr < L && rr < r1) {
                const size_t row = raw_row(i, rr);
                qw[u] = __ldg(reinterpret_cast<const uint4*>(p.q_raw + row * p.q_ld + 8 * grp));
                kw[u] = __ldg(reinterpret_cast<const uint4*>(p.k_raw + row * p.k_ld + 8 * grp));
            }
        }
    };
    // thread 0: the consumed count of the slot the next write takes
    unsigned seen = 0;
    auto peek = [&](int i) {
        if (wtid == 0 && i >= kRing && i < nchunks)
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];"
                         : "=r"(seen)
                         : "l"(p.consumed + gl * kRing + i % kRing)
                         : "memory");
    };
    uint4 aq[kBatch], ak[kBatch];   // raw rows of the next chunk to write, loaded ahead

    // This CTA's share of chunk i into the ring (the first kBatch rows of the
    // thread from aq / ak); the bulk stores are left in flight.
    auto write_share = [&](int i) -> bool {
        bool okp = true;
        if (i >= kRing && wtid == 0) {
            const unsigned need = (unsigned)(nt * (i / kRing));
            if (seen < need) okp = wait_count(p.consumed + gl * kRing + i % kRing, need);
        }
        if (!qwg_all(okp)) return false;
        const int n0 = i * kC, L = min(kC, N - n0);
        const size_t slot0 = ((size_t)gl * kRing + (size_t)(i % kRing)) * kC;   // ring row of the slot's row 0
        float cs[4], sn[4];
        const double pos = (double)(p.pos0 + n0 + r0 + rsub);
#pragma unroll
        for (int k = 0; k < 4; k++) {
            cs[k] = 1.f;
            sn[k] = 0.f;
            if (turn) __sincosf(angle_mod_2pi(pos * theta[k]), &sn[k], &cs[k]);
        }
        for (int p0 = r0; p0 < r1; p0 += kPiece) {
            const int p1 = min(p0 + kPiece, r1);
            uint8_t* stq = sQ;
            uint8_t* stk = sQ + (size_t)kPiece * DK * 2;
            // rows rb, rb + kStep, ... (kBatch of them) from qw / kw into the staging buffer
            auto put = [&](int rb, uint4 (&qw)[kBatch], uint4 (&kw)[kBatch]) {
#pragma unroll
                for (int u = 0; u < kBatch; u++) {
                    const int rr = rb + u * kStep;
                    if (rr >= p1) break;
                    uint4 qo = qw[u], ko = kw[u];
                    if (real && rr < L) {
                        // k' scale gamma^(a-r), a = min(anchor, L-1): exponent in fp64, exp2 in fp32
                        const float zeta = exp2f((float)((double)(min(anc, L - 1) - rr) * lg));
                        float ck[4], sk[4];
#pragma unroll
                        for (int k = 0; k < 4; k++) {
                            ck[k] = cs[k] * zeta;
                            sk[k] = sn[k] * zeta;
                        }
                        qo = turn_group(qo, cs, sn);
                        ko = turn_group(ko, ck, sk);
                    }
                    const size_t o = ((size_t)(rr - p0) * DK + 8 * grp) * 2;
                    *reinterpret_cast<uint4*>(stq + o) = qo;
                    *reinterpret_cast<uint4*>(stk + o) = ko;
                    if (turn) {
#pragma unroll
                        for (int k = 0; k < 4; k++) {
                            const float c2 = cs[k] * cstep[k] - sn[k] * sstep[k];
                            sn[k] = sn[k] * cstep[k] + cs[k] * sstep[k];
                            cs[k] = c2;
                        }
                    }
                }
            };
            for (int rb = p0 + rsub; rb < p1; rb += kBatch * kStep) {
                if (rb == r0 + rsub) {
                    put(rb, aq, ak);
                } else {
                    uint4 qw[kBatch], kw[kBatch];
                    load_rows(i, rb, qw, kw);
                    put(rb, qw, kw);
                }
            }
            // the staged rows go to the ring by one thread's bulk stores; the
            // staging buffer is reused once they have been read
            tc::fence_proxy_async_smem();
            qwg_all(true);
            if (wtid == 0) {
                const uint32_t bytes = (uint32_t)(p1 - p0) * DK * 2;
                tc::bulk_store(p.ring_q + (slot0 + p0) * DK, stq, bytes);
                tc::bulk_store(p.ring_k + (slot0 + p0) * DK, stk, bytes);
                tc::bulk_commit_group();
                tc::bulk_wait_group_read<0>();
            }
            qwg_all(true);
        }
        return true;
    };
    // thread 0: once the bulk stores of chunk i have completed, its count
    auto release = [&](int i) {
        if (wtid == 0) {
            tc::bulk_wait_group<0>();
            asm volatile("fence.proxy.async.global;" ::: "memory");
            count_release(p.ready + gl * kRing + i % kRing);
        }
    };

    for (int i = 0; i < kLead && i < nchunks; i++) {
        load_rows(i, r0 + rsub, aq, ak);
        if (!write_share(i)) return false;
        release(i);
    }
    // the staging buffer is the producer's from here on (qempty phase 0)
    elect_arrive(&bars.qempty, lane);
    load_rows(kLead, r0 + rsub, aq, ak);
    for (int jq = 0; jq < nchunks; jq++) {
        peek(jq + kLead);
        if (jq > 0 && !qwg_all(tc::mbar_wait(&bars.qtm, (jq - 1) & 1))) return false;
        if (!qwg_all(tc::mbar_wait(&bars.qfull, jq & 1))) return false;
        tc::tc_fence_after();
        // one slab at a time (32 registers of Q in flight)
#pragma unroll 1
        for (int g = 0; g < DK / 64; g++) {
            uint32_t w[32];
#pragma unroll
            for (int c16 = 0; c16 < 8; c16++) {
                const uint4 x = *reinterpret_cast<const uint4*>(sQ + g * (kC * 128) +
                                                                tc::sw128_off((uint32_t)r, (uint32_t)c16));
                w[4 * c16 + 0] = x.x;
                w[4 * c16 + 1] = x.y;
                w[4 * c16 + 2] = x.z;
                w[4 * c16 + 3] = x.w;
            }
            tc::tmem_st32(tb + lane_off + kTQ + 32 * g, w);
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
        elect_arrive(&bars.qready, lane);
        const int i = jq + kLead;
        if (jq > 0 && i - 1 < nchunks) release(i - 1);
        if (i < nchunks) {
            // (the staging buffer's reads above are done: the TMEM stores
            // consumed their registers, and every thread has passed them)
            qwg_all(true);
            if (!write_share(i)) return false;
        }
        // the staging buffer goes back to the producer: the generic reads and
        // writes above are ordered before its next async-proxy write
        tc::fence_proxy_async_smem();
        elect_arrive(&bars.qempty, lane);
        if (i < nchunks) load_rows(i + 1, r0 + rsub, aq, ak);
    }
    return true;
}

template <int DK, typename Tout, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1) k_chunkwise_ws(const __grid_constant__ WsParams p) {
    constexpr int kParts = DK / kPartDk;
    constexpr int kQSlabs = DK / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ Bars bars;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = p.dv / kW, jt = (int)blockIdx.x % nt;     // this CTA's 64 value columns
    const int gl = (int)blockIdx.x / nt;                      // this launch's head index
    const int h = (p.bh0 + gl) % p.H, b = (p.bh0 + gl) / p.H;
    const int j0 = jt * kW;
    const int N = p.N;
    const int nchunks = (N + kC - 1) / kC;
    const double lg = p.hc.log2g[h];
    // a head whose decay is too fast for the folded factors is computed by
    // the recurrent kernel; its CTAs (all of them, so none waits on another)
    // leave before touching anything
    if (p.hc.anchor[h] < 0) return;
    const int has_init = p.istate != nullptr;
    constexpr int kXfWarps = 8;  // transform warps arriving on the warpgroup barriers

    if (tid == 0) {
        tc::mbar_init(&bars.qfull, 1);
        tc::mbar_init(&bars.qempty, 4);
        for (int i = 0; i < kKSlots; i++) {
            tc::mbar_init(&bars.kfull[i], 1);
            tc::mbar_init(&bars.kempty[i], 2);  // read by both issuers
        }
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&bars.vfull[i], 1);
            tc::mbar_init(&bars.vempty[i], p.tma_out ? 1 : 2);
        }
        tc::mbar_init(&bars.qready, 4);
        tc::mbar_init(&bars.qtm, 1);
        tc::mbar_init(&bars.afull, 1);
        tc::mbar_init(&bars.aread, kXfWarps);
        tc::mbar_init(&bars.pready, kXfWarps);
        tc::mbar_init(&bars.dsdone, 1);
        tc::mbar_init(&bars.dsfree, kXfWarps);
        tc::mbar_init(&bars.tready, kXfWarps);
        tc::mbar_init(&bars.ofull, 1);
        tc::mbar_init(&bars.ofree, kXfWarps);
        for (int i = 0; i < 2; i++) {
            // bf16: both column halves staged at once; fp32: one half per round
            tc::mbar_init(&bars.ostaged[i], sizeof(Tout) == 2 ? kXfWarps : kXfWarps / 2);
            tc::mbar_init(&bars.ostaged2[i], kXfWarps / 2);
            tc::mbar_init(&bars.ohalf[i], 1);
        }
        s_fail = 0;
        tc::fence_barrier_init();
        tc::prefetch_tmap(&p.tq);
        tc::prefetch_tmap(&p.tk);
        tc::prefetch_tmap(&p.tv);
    }
    if (warp == 1) tc::tmem_alloc(&s_tmem, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tb = s_tmem;
    bool ok = true;

    if (warp < 4) {
        regs_dec<kRegsCtl>();
        if (warp == 0 && lane == 0) {
            // -------------------------------------------- TMA producer
            // L2 prefetch of chunk jp: the CTAs of one head split the Q and K'
            // boxes between them; each prefetches its own V tile.
            // (the fused ring is written into L2 by the CTAs themselves)
            auto prefetch = [&](int jp) {
                if (jp >= nchunks) return;
                const int n0p = jp * kC;
                if constexpr (!FUSED)
                    for (int i = jt; i < 2 * kQSlabs; i += nt)
                        tc::tma_prefetch_l2_4d(i < kQSlabs ? &p.tq : &p.tk, 64 * (i % kQSlabs), h, n0p, b);
                tc::tma_prefetch_l2_4d(&p.tv, j0, h, n0p, b);
            };
            prefetch(0);
            prefetch(1);
            for (int jc = 0; jc < nchunks && ok; jc++) {
                const int n0 = jc * kC;
                // coordinates of the chunk's rows in the q / k' tensor maps:
                // (head, token, batch), or (ring row, head of the launch, 0)
                const int c1 = FUSED ? (jc % kRing) * kC : h, c2 = FUSED ? gl : n0, c3 = FUSED ? 0 : b;
                prefetch(jc + 2);
                // (fused: the Q warpgroup hands the staging buffer over once after
                // writing its first ring rows, so chunk jc waits for phase jc)
                if (FUSED) ok = tc::mbar_wait(&bars.qempty, jc & 1);
                else if (jc > 0) ok = tc::mbar_wait(&bars.qempty, (jc - 1) & 1);
                // fused: every CTA of the head has written its share of the chunk
                if (FUSED && ok)
                    ok = wait_count(p.ready + gl * kRing + jc % kRing, (unsigned)(nt * (jc / kRing + 1)));
                if (!ok) break;
                tc::mbar_arrive_expect_tx(&bars.qfull, DK * kC * 2);
                for (int s = 0; s < kQSlabs; s++)
                    tc::tma_load_4d(sm + WsSmem<DK>::kQ + s * (kC * 128), &p.tq, &bars.qfull, 64 * s, c1, c2, c3);
                for (int part = 0; part < kParts && ok; part++) {
                    const int g = jc * kParts + part, slot = g % kKSlots, u = g / kKSlots;
                    if (u > 0) ok = tc::mbar_wait(&bars.kempty[slot], (u - 1) & 1);
                    if (!ok) break;
                    uint8_t* dst = sm + WsSmem<DK>::kK + slot * kKPartBytes;
                    tc::mbar_arrive_expect_tx(&bars.kfull[slot], kKPartBytes);
                    for (int s = 0; s < 2; s++)
                        tc::tma_load_4d(dst + s * (kC * 128), &p.tk, &bars.kfull[slot], part * kPartDk + 64 * s, c1,
                                        c2, c3);
                }
                const int vs = jc & 1;
                if (ok && jc >= 2) ok = tc::mbar_wait(&bars.vempty[vs], ((jc >> 1) & 1) ^ 1);
                if (!ok) break;
                tc::mbar_arrive_expect_tx(&bars.vfull[vs], kVBytes);
                tc::tma_load_4d(sm + WsSmem<DK>::kV + vs * kVBytes, &p.tv, &bars.vfull[vs], j0, h, n0, b);
            }
        } else if (warp == 2) {
            // ------------------------------------------ output store (bf16)
            // Each chunk's tile, staged by the transform warpgroups in the V
            // slot it used, goes out in one TMA store; the slot returns to the
            // producer once the store has read it.  One barrier per slot, so
            // the staging of chunk jc + 2 (which needs that slot's next V)
            // cannot complete a phase before this warp has seen chunk jc's.
            if (p.tma_out) {
                // the store (or add, with accumulate) of one staged tile at
                // column c0; reversed output: the tile's rows run backwards
                // from row N - n0 - 1, staged that way round
                auto put = [&](const uint8_t* slot, int c0, int jc) {
                    const int row0 = p.out_rev ? N - jc * kC - kC : jc * kC;
                    if (p.accumulate) tc::tma_reduce_add_4d(&p.to, slot, c0, h, row0, b);
                    else tc::tma_store_4d(&p.to, slot, c0, h, row0, b);
                    tc::bulk_commit_group();
                    tc::bulk_wait_group_read<0>();
                };
                for (int jc = 0; jc < nchunks && ok; jc++) {
                    const int vs = jc & 1;
                    const uint32_t par = (jc >> 1) & 1;
                    // a reversed partial last chunk would start before row 0: the
                    // transform warps store it directly
                    const bool direct = p.out_rev && jc == nchunks - 1 && N - jc * kC < kC;
                    uint8_t* slot = sm + WsSmem<DK>::kV + vs * kVBytes;
                    ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars.ostaged[vs], par));
                    if (!ok) break;
                    if (lane == 0) {
                        if (!direct) put(slot, j0, jc);
                        // fp32: the second column half goes through the same slot
                        tc::mbar_arrive(sizeof(Tout) == 2 ? &bars.vempty[vs] : &bars.ohalf[vs]);
                    }
                    __syncwarp();
                    if constexpr (sizeof(Tout) == 4) {
                        ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars.ostaged2[vs], par));
                        if (!ok) break;
                        if (lane == 0) {
                            if (!direct) put(slot, j0 + kW / 2, jc);
                            tc::mbar_arrive(&bars.vempty[vs]);
                        }
                        __syncwarp();
                    }
                }
                if (lane == 0) tc::bulk_wait_group<0>();  // the last tile is in global memory
            }
        } else if (warp == 3) {
            // ------------------------------------ state-update issuer
            const uint32_t id_st = tc::idesc_bf16_f32(128, kW, 1, 1);
            const uint64_t dk_mn = tc::sdesc_sw128(tc::smem_u32(sm + WsSmem<DK>::kK), kC * 128, 1024);
            const uint64_t dv_mn = tc::sdesc_sw128(tc::smem_u32(sm + WsSmem<DK>::kV), kC * 128, 1024);
            auto wait = [&](uint64_t* bar, uint32_t parity) {
                return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity));
            };
            for (int jc = 0; jc < nchunks && ok; jc++) {
                const uint32_t vo = (uint32_t)((jc & 1) * kVBytes) >> 4;
                ok = wait(&bars.vfull[jc & 1], (jc >> 1) & 1);
                if (ok && jc > 0) ok = wait(&bars.dsfree, (jc - 1) & 1);
                if (!ok) break;
                tc::tc_fence_after();
                for (int part = 0; part < kParts && ok; part++) {
                    const int g = jc * kParts + part, slot = g % kKSlots, u = g / kKSlots;
                    ok = wait(&bars.kfull[slot], u & 1);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const uint32_t ko = (uint32_t)(slot * kKPartBytes) >> 4;
#pragma unroll
                    for (int k = 0; k < kC / 16; k++)
                        tc::mma_bf16_ss_elect(tb + kTD + part * kW, dk_mn + ko + (uint32_t)((k * 2048) >> 4),
                                              dv_mn + vo + (uint32_t)((k * 2048) >> 4), id_st, k > 0);
                    tc::mma_commit_elect(&bars.kempty[slot]);
                }
                if (!ok) break;
                tc::mma_commit_elect(&bars.dsdone);
                if (!p.tma_out) tc::mma_commit_elect(&bars.vempty[jc & 1]);
            }
        } else if (warp == 1) {
            // --------------------------------------------- tensor pipe
            // The whole warp walks the loop (warp-uniform descriptors); one
            // elected lane issues each tcgen05 instruction.
            const uint32_t id_qk = tc::idesc_bf16_f32(128, 128, 0, 0);
            const uint32_t id_qt = tc::idesc_bf16_f32(128, kW, 0, 1);
            const uint32_t id_pv = tc::idesc_bf16_f32(128, kW, 0, 1);
            // descriptor bases; offsets are added in 16-byte units
            const uint64_t dk_k = tc::sdesc_sw128(tc::smem_u32(sm + WsSmem<DK>::kK), 16, 1024);         // K' as B, K-major
            const uint64_t dv_mn = tc::sdesc_sw128(tc::smem_u32(sm + WsSmem<DK>::kV), kC * 128, 1024);  // V as B, MN-major
            const uint64_t dt_mn = tc::sdesc_sw128(tc::smem_u32(sm + WsSmem<DK>::kT), DK * 128, 1024);  // T as B, MN-major
            // a timed-out wait must leave the warp converged for elect.sync
            auto wait = [&](uint64_t* bar, uint32_t parity) {
                return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity));
            };
            // Per chunk: A = Q K'^T part by part with dS = K'^T V of every part
            // but the last right behind it (so each K' part is released early),
            // then the read-out O = Q T, the last dS part, and O += P V.
            for (int jc = 0; jc < nchunks && ok; jc++) {
                const uint32_t vo = (uint32_t)((jc & 1) * kVBytes) >> 4;
                ok = wait(&bars.qready, jc & 1);
                if (ok && jc > 0) ok = wait(&bars.aread, (jc - 1) & 1);
                if (!ok) break;
                for (int part = 0; part < kParts && ok; part++) {
                    const int g = jc * kParts + part, slot = g % kKSlots, u = g / kKSlots;
                    ok = wait(&bars.kfull[slot], u & 1);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const uint32_t ko = (uint32_t)(slot * kKPartBytes) >> 4;
#pragma unroll
                    for (int k = 0; k < kPartDk / 16; k++)
                        tc::mma_bf16_ts_elect(tb + kTA, tb + kTQ + 64 * part + 8 * k,
                                              dk_k + ko + (uint32_t)(((k / 4) * (kC * 128) + (k % 4) * 32) >> 4),
                                              id_qk, (part > 0) || (k > 0));
                    tc::mma_commit_elect(&bars.kempty[slot]);
                }
                if (!ok) break;
                tc::mma_commit_elect(&bars.afull);
                // ---- O = Q T  (read-out of the state before this chunk; none for
                // the first chunk unless the call continues from a given state)
                if (jc > 0 || has_init) {
                    ok = wait(&bars.tready, (jc - 1 + has_init) & 1);
                    if (ok && jc > 0) ok = wait(&bars.ofree, (jc - 1) & 1);
                    if (!ok) break;
                    tc::tc_fence_after();
#pragma unroll 4
                    for (int k = 0; k < DK / 16; k++)
                        tc::mma_bf16_ts_elect(tb + kTO, tb + kTQ + 8 * k, dt_mn + (uint32_t)((16 * k * 128) >> 4),
                                              id_qt, k > 0);
                }
                tc::mma_commit_elect(&bars.qtm);  // Q in TMEM and T in smem are read
                // ---- O += P V  (P from TMEM; V of this chunk must have landed:
                // nothing else this warp waits on implies it, since the
                // producer loads V after the chunk's K' parts)
                ok = wait(&bars.pready, jc & 1);
                if (ok) ok = wait(&bars.vfull[jc & 1], (jc >> 1) & 1);
                if (!ok) break;
                tc::tc_fence_after();
#pragma unroll
                for (int k = 0; k < kC / 16; k++)
                    tc::mma_bf16_ts_elect(tb + kTO, tb + kTP + 8 * k, dv_mn + vo + (uint32_t)((k * 2048) >> 4), id_pv,
                                          (jc > 0) || has_init || (k > 0));
                tc::mma_commit_elect(&bars.ofull);
                // with the TMA-store epilogue the output tile is staged in this
                // V slot, which the epilogue hands back once the store has read it
                if (!p.tma_out) tc::mma_commit_elect(&bars.vempty[jc & 1]);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------- Q warpgroup
        // Thread r copies row r of the next chunk's Q from the staging buffer
        // into registers as soon as it lands (freeing the buffer for the
        // chunk after), and writes it into TMEM columns [kTQ, kTQ + DK/2)
        // once the read-out of the current chunk has consumed the previous
        // one.  Rows past the end arrive as zeros from the TMA fill.
        regs_inc<kRegsQ>();
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint8_t* sQ = sm + WsSmem<DK>::kQ;
        uint4 qv[DK / 8];
        if constexpr (FUSED) {
            ok = q_role_fused<DK>(p, const_cast<uint8_t*>(sQ), tb, lane_off, r, quarter, lane, nt, jt, gl, b, h,
                                  nchunks, lg, p.hc.anchor[h], bars);
        } else
        for (int jq = 0; jq < nchunks && ok; jq++) {
            ok = tc::mbar_wait(&bars.qfull, jq & 1);
            if (!ok) break;
#pragma unroll
            for (int s = 0; s < kQSlabs; s++)
#pragma unroll
                for (int c16 = 0; c16 < 8; c16++)
                    qv[8 * s + c16] = *reinterpret_cast<const uint4*>(sQ + s * (kC * 128) +
                                                                      tc::sw128_off((uint32_t)r, (uint32_t)c16));
            // The buffer is handed back to the TMA only once every load has
            // landed in registers: an arrive right behind the loads can let
            // the next tile's bulk copy overwrite data a load has not read
            // yet.  Consuming one word of each load makes the warp wait for
            // them; the proxy fence orders them before the async-proxy write.
            {
                uint32_t dep = 0;
#pragma unroll
                for (int i = 0; i < DK / 8; i++) dep ^= qv[i].x;
                asm volatile("" ::"r"(dep));
            }
            tc::fence_proxy_async_smem();
            elect_arrive(&bars.qempty, lane);
            if (jq > 0) ok = tc::mbar_wait(&bars.qtm, (jq - 1) & 1);
            if (!ok) break;
            tc::tc_fence_after();
#pragma unroll
            for (int g = 0; g < DK / 64; g++) {
                uint32_t w[32];
#pragma unroll
                for (int k = 0; k < 8; k++) {
                    w[4 * k + 0] = qv[8 * g + k].x;
                    w[4 * k + 1] = qv[8 * g + k].y;
                    w[4 * k + 2] = qv[8 * g + k].z;
                    w[4 * k + 3] = qv[8 * g + k].w;
                }
                tc::tmem_st32(tb + lane_off + kTQ + 32 * g, w);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            elect_arrive(&bars.qready, lane);
        }
    } else {
        // ------------------------------------------ transform warpgroups
        // Warps 8-11 and 12-15 form two warpgroups; each covers TMEM lanes
        // 0..127 (a warp reaches the lane quarter warp % 4) and takes one half
        // of the columns of every phase.  The fp32 state R lives in their
        // registers: row r of every 128-row block, 32 columns each.
        regs_inc<kRegsXf>();
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter ..
        const int wg = (warp - 8) >> 2;               // column half
        const int r = quarter * 32 + lane;            // chunk row / state row in a block
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        uint8_t* sT = sm + WsSmem<DK>::kT;
        float R[kParts][32];
        // decay powers of a full chunk and of the (possibly shorter) last one:
        // state decay gamma^L, row scale gamma^(r-a), read-out copy gamma^(a+1),
        // and gamma^(L-1-a) on dS (exactly 1 when a = L-1)
        // (the last chunk's are evaluated where they are used, once)
        const int L_last = N - (nchunks - 1) * kC;
        const int a_full = p.hc.anchor[h], a_last = min(a_full, L_last - 1);
        auto pw = [&](int e) { return (float)exp2((double)e * lg); };
        const float g_full = pw(kC), sc_full = pw(r - a_full), t_full = pw(a_full + 1), f_full = pw(kC - 1 - a_full);
        if (has_init) {
            // Continue from the given state: R = S_init, and the first read-out
            // uses T = gamma^(a0+1) S_init (a0 the first chunk's anchor).
            const float g0 = nchunks == 1 ? pw(a_last + 1) : t_full;
#pragma unroll
            for (int part = 0; part < kParts; part++) {
                const int dr = part * kPartDk + r;
                const float4* src = reinterpret_cast<const float4*>(p.istate + (((size_t)b * p.H + h) * p.dks + dr) * p.dv +
                                                                    j0 + 32 * wg);
#pragma unroll
                for (int c4 = 0; c4 < 8; c4++) {
                    // rows past the caller's d_k (padding) start at zero
                    const float4 x = dr < p.dks ? __ldg(src + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
                    R[part][4 * c4 + 0] = x.x;
                    R[part][4 * c4 + 1] = x.y;
                    R[part][4 * c4 + 2] = x.z;
                    R[part][4 * c4 + 3] = x.w;
                }
#pragma unroll
                for (int c4 = 0; c4 < 4; c4++) {
                    const int base = c4 * 8;
                    uint4 v;
                    v.x = tc::pack_bf16x2(g0 * R[part][base + 0], g0 * R[part][base + 1]);
                    v.y = tc::pack_bf16x2(g0 * R[part][base + 2], g0 * R[part][base + 3]);
                    v.z = tc::pack_bf16x2(g0 * R[part][base + 4], g0 * R[part][base + 5]);
                    v.w = tc::pack_bf16x2(g0 * R[part][base + 6], g0 * R[part][base + 7]);
                    *reinterpret_cast<uint4*>(sT + tc::sw128_off((uint32_t)dr, (uint32_t)(4 * wg + c4))) = v;
                }
            }
            tc::fence_proxy_async_smem();
            elect_arrive(&bars.tready, lane);
        } else {
#pragma unroll
            for (int part = 0; part < kParts; part++)
#pragma unroll
                for (int i = 0; i < 32; i++) R[part][i] = 0.f;
        }

        for (int jc = 0; jc < nchunks && ok; jc++) {
            const int n0 = jc * kC, L = min(kC, N - n0);
            const bool last = (jc == nchunks - 1);
            // the row's normalization factor, loaded now and used by the epilogue
            const float rs = (p.rowscale && r < L) ? __ldg(p.rowscale + ((size_t)b * N + n0 + r) * p.H + h) : 1.f;
            // ---- mask: P = tril(A) as packed bf16 into TMEM, 32 A columns at a time
            ok = tc::mbar_wait(&bars.afull, jc & 1);
            if (!ok) break;
            // fused: every load of this chunk from the ring has landed (A read
            // all of Q and K'), so the slot may be rewritten as far as this CTA goes
            if constexpr (FUSED)
                if (warp == 8 && lane == 0) count_release(p.consumed + gl * kRing + jc % kRing);
            tc::tc_fence_after();
            {
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    uint32_t a[32], w[16];
                    tc::tmem_ld32(tb + lane_off + kTA + 64 * wg + 32 * hh, a);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const int c = 64 * wg + 32 * hh + 2 * i;
                        const float lo = (c <= r) ? __uint_as_float(a[2 * i]) : 0.f;
                        const float hi = (c + 1 <= r) ? __uint_as_float(a[2 * i + 1]) : 0.f;
                        w[i] = tc::pack_bf16x2(lo, hi);
                    }
                    tc::tmem_st16(tb + lane_off + kTP + 32 * wg + 16 * hh, w);
                }
                tc::tc_fence_before();
                elect_arrive(&bars.aread, lane);
                tc::tmem_st_wait();
            }
            tc::tc_fence_before();
            elect_arrive(&bars.pready, lane);
            // ---- state: R = gamma^L R + dS; T = gamma^L_next R (bf16, read-out of the next chunk)
            ok = tc::mbar_wait(&bars.dsdone, jc & 1);
            if (!ok) break;
            tc::tc_fence_after();
            {
                const float gL = last ? pw(L_last) : g_full, fD = last ? pw(L_last - 1 - a_last) : f_full;
#pragma unroll
                for (int part = 0; part < kParts; part++) {
                    uint32_t d[32];
                    tc::tmem_ld32(tb + lane_off + kTD + part * kW + 32 * wg, d);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; i++) R[part][i] = fmaf(gL, R[part][i], fD * __uint_as_float(d[i]));
                }
                tc::tc_fence_before();
                elect_arrive(&bars.dsfree, lane);
                if (!last) {
                    const float gN = (jc + 1 == nchunks - 1) ? pw(a_last + 1) : t_full;
                    // T is overwritten only once this chunk's read-out has consumed it
                    ok = tc::mbar_wait(&bars.qtm, jc & 1);
                    if (!ok) break;
#pragma unroll
                    for (int part = 0; part < kParts; part++) {
                        const int dr = part * kPartDk + r;
#pragma unroll
                        for (int c4 = 0; c4 < 4; c4++) {
                            const int base = c4 * 8;
                            uint4 v;
                            v.x = tc::pack_bf16x2(gN * R[part][base + 0], gN * R[part][base + 1]);
                            v.y = tc::pack_bf16x2(gN * R[part][base + 2], gN * R[part][base + 3]);
                            v.z = tc::pack_bf16x2(gN * R[part][base + 4], gN * R[part][base + 5]);
                            v.w = tc::pack_bf16x2(gN * R[part][base + 6], gN * R[part][base + 7]);
                            *reinterpret_cast<uint4*>(sT + tc::sw128_off((uint32_t)dr, (uint32_t)(4 * wg + c4))) = v;
                        }
                    }
                    tc::fence_proxy_async_smem();
                    elect_arrive(&bars.tready, lane);
                } else if (p.fstate) {
#pragma unroll
                    for (int part = 0; part < kParts; part++) {
                        const int dr = part * kPartDk + r;
                        if (dr >= p.dks) continue;  // padding rows are not part of the state
                        float4* dst = reinterpret_cast<float4*>(p.fstate + (((size_t)b * p.H + h) * p.dks + dr) * p.dv +
                                                                j0 + 32 * wg);
#pragma unroll
                        for (int c4 = 0; c4 < 8; c4++)
                            dst[c4] = make_float4(R[part][4 * c4], R[part][4 * c4 + 1], R[part][4 * c4 + 2],
                                                  R[part][4 * c4 + 3]);
                    }
                }
            }
            // ---- epilogue: out = gamma^(r+1-L) O
            ok = tc::mbar_wait(&bars.ofull, jc & 1);
            if (!ok) break;
            tc::tc_fence_after();
            {
                uint32_t o[32];
                tc::tmem_ld32(tb + lane_off + kTO + 32 * wg, o);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                elect_arrive(&bars.ofree, lane);
                if constexpr (sizeof(Tout) == 2) {
                    if (p.tma_out) {
                        // Stage the bf16 tile in the V slot of this chunk (free since
                        // P V completed) in the TMA's 128-byte swizzle, then one
                        // thread stores it: rows past N are clipped by the TMA.
                        uint8_t* sO = sm + WsSmem<DK>::kV + (jc & 1) * kVBytes;
                        const float sc = (last ? pw(r - a_last) : sc_full) * rs;
#pragma unroll
                        for (int c16 = 0; c16 < 4; c16++) {
                            const int base = c16 * 8;
                            uint4 v;
                            v.x = tc::pack_bf16x2(__uint_as_float(o[base + 0]) * sc, __uint_as_float(o[base + 1]) * sc);
                            v.y = tc::pack_bf16x2(__uint_as_float(o[base + 2]) * sc, __uint_as_float(o[base + 3]) * sc);
                            v.z = tc::pack_bf16x2(__uint_as_float(o[base + 4]) * sc, __uint_as_float(o[base + 5]) * sc);
                            v.w = tc::pack_bf16x2(__uint_as_float(o[base + 6]) * sc, __uint_as_float(o[base + 7]) * sc);
                            *reinterpret_cast<uint4*>(sO + tc::sw128_off((uint32_t)r, (uint32_t)(4 * wg + c16))) = v;
                        }
                        tc::fence_proxy_async_smem();
                        elect_arrive(&bars.ostaged[jc & 1], lane);
                        continue;
                    }
                } else {
                    if (p.tma_out) {
                        // fp32: column half wg of the tile, one half at a time
                        // through the V slot (the second waits for the first
                        // to be read by its store); reversed output stages row r
                        // at 127 - r.  A reversed partial last chunk is stored
                        // directly below, the store warp only told it is staged.
                        const bool direct = p.out_rev && last && L < kC;
                        if (!direct) {
                            uint8_t* sO = sm + WsSmem<DK>::kV + (jc & 1) * kVBytes;
                            const float sc = (last ? pw(r - a_last) : sc_full) * rs;
                            const uint32_t srow = p.out_rev ? (uint32_t)(kC - 1 - r) : (uint32_t)r;
                            if (wg == 1) {
                                ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars.ohalf[jc & 1], (jc >> 1) & 1));
                                if (!ok) break;
                            }
#pragma unroll
                            for (int c4 = 0; c4 < 8; c4++) {
                                const float4 y = make_float4(
                                    __uint_as_float(o[4 * c4 + 0]) * sc, __uint_as_float(o[4 * c4 + 1]) * sc,
                                    __uint_as_float(o[4 * c4 + 2]) * sc, __uint_as_float(o[4 * c4 + 3]) * sc);
                                *reinterpret_cast<float4*>(sO + tc::sw128_off(srow, (uint32_t)c4)) = y;
                            }
                            tc::fence_proxy_async_smem();
                            elect_arrive(wg == 0 ? &bars.ostaged[jc & 1] : &bars.ostaged2[jc & 1], lane);
                            continue;
                        }
                        elect_arrive(wg == 0 ? &bars.ostaged[jc & 1] : &bars.ostaged2[jc & 1], lane);
                    }
                }
                if (r < L) {
                    const float sc = (last ? pw(r - a_last) : sc_full) * rs;
                    const int n = p.out_rev ? N - 1 - (n0 + r) : n0 + r;
                    Tout* dst = reinterpret_cast<Tout*>(p.out) + (((size_t)b * N + n) * p.H + h) * p.dv + j0 + 32 * wg;
                    if constexpr (sizeof(Tout) == 2) {
#pragma unroll
                        for (int c16 = 0; c16 < 4; c16++) {
                            const int base = c16 * 8;
                            uint4 v;
                            v.x = tc::pack_bf16x2(__uint_as_float(o[base + 0]) * sc, __uint_as_float(o[base + 1]) * sc);
                            v.y = tc::pack_bf16x2(__uint_as_float(o[base + 2]) * sc, __uint_as_float(o[base + 3]) * sc);
                            v.z = tc::pack_bf16x2(__uint_as_float(o[base + 4]) * sc, __uint_as_float(o[base + 5]) * sc);
                            v.w = tc::pack_bf16x2(__uint_as_float(o[base + 6]) * sc, __uint_as_float(o[base + 7]) * sc);
                            reinterpret_cast<uint4*>(dst)[c16] = v;
                        }
                    } else {
#pragma unroll
                        for (int c4 = 0; c4 < 8; c4++) {
                            float4 y = make_float4(__uint_as_float(o[4 * c4 + 0]) * sc, __uint_as_float(o[4 * c4 + 1]) * sc,
                                                   __uint_as_float(o[4 * c4 + 2]) * sc, __uint_as_float(o[4 * c4 + 3]) * sc);
                            if (p.accumulate) {
                                const float4 x = reinterpret_cast<const float4*>(dst)[c4];
                                y.x += x.x;
                                y.y += x.y;
                                y.z += x.z;
                                y.w += x.w;
                            }
                            reinterpret_cast<float4*>(dst)[c4] = y;
                        }
                    }
                }
            }
        }
    }

    if (!ok) atomicExch(&s_fail, 1);
    tc::tc_fence_before();
    __syncthreads();
    if (s_fail && tid == 0) atomicExch(&g_err_chunk_ws, kErrTimeout);
    if (warp == 1) tc::tmem_dealloc(tb, 512);
}

template <int DK, typename Tout>
ret_status launch_main(const WsParams& p, cudaStream_t s) {
    auto kern = k_chunkwise_ws<DK, Tout, false>;
    const int smem = (int)WsSmem<DK>::kBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return check_launch("chunkwise (workspace path): smem attribute");
    kern<<<p.nmain, kThreads, smem, s>>>(p);
    return check_launch("chunkwise (workspace path)");
}

}  // namespace

// Self-test of the bounded wait: one thread waits on an mbarrier that
// nothing arrives on, with the wait the kernels use, gives up after `polls`
// polls and records the timeout in the device error word as they do.
__global__ void k_wait_selftest(uint32_t polls) {
    __shared__ uint64_t bar;
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
    if (!tc::mbar_wait(&bar, 0, polls)) atomicExch(&g_err_chunk_ws, kErrTimeout);
}

ret_status launch_wait_selftest(uint32_t polls, cudaStream_t s) {
    k_wait_selftest<<<1, 1, 0, s>>>(polls);
    return check_launch("bounded-wait self-test");
}

// The workspace holds a copy of q (q_rot) when the queries are rotated or
// padded to the kernel's d_k.
static bool q_copied(const RetArgs& a) { return a.xpos || (a.dk_real && a.dk_real != a.dk); }

// Workspace layout: k' [B, N, H, dk] bf16, then q_rot (rotated or padded q).
size_t chunkwise_ws_bytes(const RetArgs& a) {
    const size_t qk = (size_t)a.B * a.N * a.H * a.dk * 2;
    return q_copied(a) ? 2 * qk : qk;
}

bool chunkwise_ws_shape_ok(const RetArgs& a) {
    if (a.in_dt != RET_BF16) return false;
    if (a.chunk != kC || !(a.dk == 128 || a.dk == 256) || a.dv % kW != 0) return false;
    if (a.N > (1 << 30)) return false;
    if ((long long)a.B * a.H * (a.dv / kW) > (1ll << 30)) return false;
    return true;
}

int chunkwise_heads_below(const RetArgs& a, int min_anchor) {
    int n = 0;
    for (int h = 0; h < a.H; h++) n += a.hc.anchor[h] < min_anchor;
    return n;
}

bool chunkwise_ws_supported(const RetArgs& a) {
    return chunkwise_ws_shape_ok(a) && chunkwise_heads_below(a, 0) == 0;
}

// Tensor maps and per-launch fields shared by both kernel variants.
static ret_status fill_params(WsParams* p, const RetArgs& a, const void* q_src, int q_pitch, const void* k_prime) {
    memset(p, 0, sizeof(*p));
    const uint64_t B = a.B, N = a.N, H = a.H, dk = a.dk, dv = a.dv, qp = (uint64_t)q_pitch;
    const uint64_t dq[4] = {dk, H, N, B};
    const uint64_t sq[3] = {dk * 2, H * dk * 2, N * H * dk * 2};
    const uint64_t sqq[3] = {qp * 2, H * qp * 2, N * H * qp * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)kC, 1};
    const uint64_t dvv[4] = {dv, H, N, B};
    const uint64_t svv[3] = {dv * 2, H * dv * 2, N * H * dv * 2};
    if (!make_tmap_bf16(&p->tq, q_src, 4, dq, sqq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_bf16(&p->tk, k_prime, 4, dq, sq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_bf16(&p->tv, a.v, 4, dvv, svv, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return RET_ERR_CUDA;
    p->out = a.out;
    p->fstate = a.final_state;
    p->istate = a.initial_state;
    p->N = a.N;
    p->H = a.H;
    p->dv = a.dv;
    p->hc = a.hc;
    p->nmain = a.B * a.H * (a.dv / kW);
    p->accumulate = a.accumulate;
    p->out_rev = a.out_rev;
    p->dks = a.dk_real ? a.dk_real : a.dk;
    p->rowscale = a.rowscale;
    p->tma_out = 0;
    // bf16 out: plain stores only; fp32 out: stores or adds, rows forward or reversed
    if (a.out_dt == RET_F32 || (!a.accumulate && !a.out_rev)) {
        if (a.out_dt == RET_BF16) {
            if (!make_tmap_bf16(&p->to, a.out, 4, dvv, svv, box, CU_TENSOR_MAP_SWIZZLE_128B)) return RET_ERR_CUDA;
        } else {
            const uint64_t sf[3] = {dv * 4, H * dv * 4, N * H * dv * 4};
            const uint32_t bf[4] = {(uint32_t)kW / 2, 1, (uint32_t)kC, 1};
            if (!make_tmap_f32(&p->to, a.out, 4, dvv, sf, bf, CU_TENSOR_MAP_SWIZZLE_128B)) return RET_ERR_CUDA;
        }
        p->tma_out = 1;
    }
    return RET_OK;
}

// ------------------------------------------------------ fused rotation
//
// The CTAs of one head wait on one another's ring writes, so a launch holds
// no more heads than can be resident at once; it is launched cooperatively,
// which makes the runtime refuse (rather than run) a grid that could not be
// co-resident.  Larger problems run as several launches, one per group of
// heads, on the same scratch.

constexpr int kFusedCtaCap = 148;   // CTAs the scratch of one launch is sized for (one per SM of a B200)

static int fused_group_cap(const RetArgs& a) {
    const int nt = a.dv / kW;
    const long long bh = (long long)a.B * a.H;
    return (int)std::min<long long>(bh, std::max(1, kFusedCtaCap / nt));
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch: ready[G][kRing], consumed[G][kRing] (u32), then the q and k'
// rings, [G, kRing, 128, dk] bf16 each.
static size_t fused_counter_bytes(size_t G) { return align256(2 * G * kRing * sizeof(unsigned)); }

size_t chunkwise_fused_bytes(const RetArgs& a) {
    const size_t G = (size_t)fused_group_cap(a);
    return fused_counter_bytes(G) + 2 * G * kRing * kC * (size_t)a.dk * 2;
}

template <int DK, typename Tout>
ret_status launch_fused(const WsParams& p, int grid, cudaStream_t s) {
    auto kern = k_chunkwise_ws<DK, Tout, true>;
    const int smem = (int)WsSmem<DK>::kBytes;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return check_launch("chunkwise (fused): smem attribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "chunkwise (fused): launch: %s", cudaGetErrorString(e));
    return check_launch("chunkwise (fused)");
}

// CTAs of the fused kernel that fit on the current device at once.
template <int DK, typename Tout>
static int fused_resident(int* out) {
    auto kern = k_chunkwise_ws<DK, Tout, true>;
    const int smem = (int)WsSmem<DK>::kBytes;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) != cudaSuccess)
        return 0;
    *out = per_sm * sms;
    return 1;
}

ret_status launch_chunkwise_fused(const RetArgs& a, void* scratch, cudaStream_t s) {
    const int nt = a.dv / kW;
    const bool f32 = a.out_dt == RET_F32;
    int resident = 0;
    const int okr = a.dk == 256 ? (f32 ? fused_resident<256, float>(&resident) : fused_resident<256, __nv_bfloat16>(&resident))
                                : (f32 ? fused_resident<128, float>(&resident) : fused_resident<128, __nv_bfloat16>(&resident));
    if (!okr) return fail(RET_ERR_CUDA, "chunkwise (fused): occupancy query failed");
    const int cap = fused_group_cap(a);
    const int G = std::min(cap, resident / nt);
    if (G < 1) return fail(RET_ERR_UNSUPPORTED, "chunkwise (fused): no room for the %d CTAs of one head", nt);
    unsigned* ctr = reinterpret_cast<unsigned*>(scratch);
    __nv_bfloat16* ring_q =
        reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(scratch) + fused_counter_bytes((size_t)cap));
    __nv_bfloat16* ring_k = ring_q + (size_t)cap * kRing * kC * a.dk;
    // the tensor maps of q and k' read the rings: {dk, ring rows, head of the launch, 1}
    WsParams p;
    ret_status st = fill_params(&p, a, a.q, a.dk, a.k);
    if (st != RET_OK) return st;
    {
        const uint64_t dk = a.dk, rows = (uint64_t)kRing * kC;
        const uint64_t dr[4] = {dk, rows, (uint64_t)cap, 1};
        const uint64_t sr[3] = {dk * 2, rows * dk * 2, (uint64_t)cap * rows * dk * 2};
        const uint32_t box[4] = {64, (uint32_t)kC, 1, 1};
        if (!make_tmap_bf16(&p.tq, ring_q, 4, dr, sr, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_bf16(&p.tk, ring_k, 4, dr, sr, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return RET_ERR_CUDA;
    }
    const int dkr = a.dk_real ? a.dk_real : a.dk;
    p.q_raw = reinterpret_cast<const __nv_bfloat16*>(a.q);
    p.k_raw = reinterpret_cast<const __nv_bfloat16*>(a.k);
    p.q_ld = a.q_ld ? a.q_ld : dkr;
    p.k_ld = a.k_ld ? a.k_ld : dkr;
    p.ring_q = ring_q;
    p.ring_k = ring_k;
    p.ready = ctr;
    p.consumed = ctr + (size_t)cap * kRing;
    p.xpos = a.xpos;
    p.pos0 = a.pos_offset;
    p.log2base = log2(a.theta_base);
    const int BH = a.B * a.H;
    for (int bh0 = 0; bh0 < BH; bh0 += G) {
        const int g = std::min(G, BH - bh0);
        p.bh0 = bh0;
        p.nmain = g * nt;
        cudaError_t e = cudaMemsetAsync(ctr, 0, 2 * (size_t)cap * kRing * sizeof(unsigned), s);
        if (e != cudaSuccess) return fail(RET_ERR_CUDA, "chunkwise (fused): counter reset: %s", cudaGetErrorString(e));
        if (a.dk == 256) st = f32 ? launch_fused<256, float>(p, g * nt, s) : launch_fused<256, __nv_bfloat16>(p, g * nt, s);
        else st = f32 ? launch_fused<128, float>(p, g * nt, s) : launch_fused<128, __nv_bfloat16>(p, g * nt, s);
        if (st != RET_OK) return st;
    }
    return RET_OK;
}

// The fused path on scratch from a stream-ordered pool the library keeps per
// device (created on the first call, never trimmed): allocated and freed in
// stream order around the launches, so concurrent calls on other streams get
// their own scratch.
ret_status launch_chunkwise_fused_pooled(const RetArgs& a, cudaStream_t s) {
    constexpr int kMaxDev = 64;
    static cudaMemPool_t pools[kMaxDev] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "chunkwise: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDev) return fail(RET_ERR_UNSUPPORTED, "chunkwise: device %d out of range", dev);
    cudaMemPool_t pool;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!pools[dev]) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            e = cudaMemPoolCreate(&pools[dev], &props);
            if (e != cudaSuccess) {
                pools[dev] = nullptr;
                return fail(RET_ERR_CUDA, "chunkwise: scratch pool: %s", cudaGetErrorString(e));
            }
            uint64_t keep = ~0ull;
            cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &keep);
        }
        pool = pools[dev];
    }
    void* scratch = nullptr;
    e = cudaMallocFromPoolAsync(&scratch, chunkwise_fused_bytes(a), pool, s);
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "chunkwise: scratch: %s", cudaGetErrorString(e));
    const ret_status st = launch_chunkwise_fused(a, scratch, s);
    e = cudaFreeAsync(scratch, s);
    if (st != RET_OK) return st;
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "chunkwise: scratch release: %s", cudaGetErrorString(e));
    return RET_OK;
}

ret_status launch_chunkwise_main(const RetArgs& a, const void* q_src, int q_pitch, const void* k_prime,
                                 cudaStream_t s) {
    WsParams p;
    ret_status st = fill_params(&p, a, q_src, q_pitch, k_prime);
    if (st != RET_OK) return st;
    const bool f32 = a.out_dt == RET_F32;
    if (a.dk == 256) return f32 ? launch_main<256, float>(p, s) : launch_main<256, __nv_bfloat16>(p, s);
    return f32 ? launch_main<128, float>(p, s) : launch_main<128, __nv_bfloat16>(p, s);
}

// Pointers into the workspace: k' first, then q_rot (rotated or padded q).
static void ws_parts(const RetArgs& a, void* ws, __nv_bfloat16** k_out, __nv_bfloat16** q_rot) {
    const size_t qk = (size_t)a.B * a.N * a.H * a.dk;
    *k_out = reinterpret_cast<__nv_bfloat16*>(ws);
    *q_rot = q_copied(a) ? *k_out + qk : nullptr;
}

ret_status launch_chunkwise_prep(const RetArgs& a, void* ws, cudaStream_t s) {
    __nv_bfloat16 *k_out, *q_rot;
    ws_parts(a, ws, &k_out, &q_rot);
    const int blocks = (int)(((long long)a.B * a.N + 7) / 8);
    const double lb = log2(a.theta_base);
    const int dkr = a.dk_real ? a.dk_real : a.dk, qcopy = q_copied(a) ? 1 : 0;
    const int qld = a.q_ld ? a.q_ld : dkr, kld = a.k_ld ? a.k_ld : dkr;
    if (a.dk == 256)
        k_prep_qk<256><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, q_rot, k_out,
                                               a.hc, a.B, a.N, a.H, a.chunk, a.xpos, a.pos_offset, lb, qld, kld, dkr,
                                               qcopy);
    else
        k_prep_qk<128><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, q_rot, k_out,
                                               a.hc, a.B, a.N, a.H, a.chunk, a.xpos, a.pos_offset, lb, qld, kld, dkr,
                                               qcopy);
    return check_launch("chunkwise (workspace path): prep");
}

ret_status launch_chunkwise_prepared(const RetArgs& a, void* ws, cudaStream_t s) {
    __nv_bfloat16 *k_out, *q_rot;
    ws_parts(a, ws, &k_out, &q_rot);
    // q_rot in the workspace is contiguous; a raw q keeps its row pitch
    const bool qc = q_copied(a);
    return launch_chunkwise_main(a, qc ? (const void*)q_rot : a.q, qc || !a.q_ld ? a.dk : a.q_ld, k_out, s);
}

ret_status launch_chunkwise_ws(const RetArgs& a, void* ws, cudaStream_t s) {
    ret_status st = launch_chunkwise_prep(a, ws, s);
    if (st != RET_OK) return st;
    return launch_chunkwise_prepared(a, ws, s);
}

// ------------------------------------------------- allocation-free variant
//
// For callers that cannot allocate device memory at call time (for example a
// plug-in running inside a host framework that owns all device memory and
// hands out no allocator, or a deployment that fixes its memory footprint at
// start-up and forbids allocation afterwards), the workspace path can run on
// a file-scope device array instead of a caller-provided buffer.  Every GPU
// that loads the library holds this array until the process exits.

constexpr size_t kStaticWsBytes = 64ull << 20;  // 64 MiB
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];

size_t chunkwise_static_ws_bytes() { return kStaticWsBytes; }

// Device address of g_static_ws in the current context, looked up once per
// device and context (the host-side symbol is only a stand-in for the device
// address).  The cache is keyed on the context as well as the device index:
// after a cudaDeviceReset the runtime makes a new primary context with the
// module loaded afresh, and the address is looked up again.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CUcontext current_context() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

static ret_status static_ws_address(void** out) {
    constexpr int kMaxDev = 64;
    static void* addr[kMaxDev] = {};
    static CUcontext ctx[kMaxDev] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "static workspace: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDev) return fail(RET_ERR_UNSUPPORTED, "static workspace: device %d out of range", dev);
    // (a thread that has made no runtime call yet has no current context:
    // the lookup below binds the device's primary context)
    const CUcontext c = current_context();
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || !c || ctx[dev] != c) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess || !p)
            return fail(RET_ERR_CUDA, "static workspace: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        addr[dev] = p;
        ctx[dev] = current_context();
    }
    *out = addr[dev];
    return RET_OK;
}

ret_status launch_chunkwise_static(const RetArgs& a, cudaStream_t s) {
    const size_t need = chunkwise_ws_bytes(a);
    if (need > kStaticWsBytes) {
        // a d_k below the kernel's is padded to it, with the queries always copied
        const int dkc = a.dk_real ? a.dk_real : a.dk;
        return fail(RET_ERR_INVALID_ARG,
                    "ret_forward_chunkwise_noalloc: this problem needs %zu bytes of scratch, above the fixed %zu "
                    "(B*N*H*%d*%d bytes for d_k = %d%s must not exceed it)",
                    need, kStaticWsBytes, a.dk, q_copied(a) ? 4 : 2, dkc,
                    a.dk_real && a.dk_real != a.dk ? ", padded to the kernel's d_k" : (a.xpos ? " with xpos" : ""));
    }
    void* ws = nullptr;
    ret_status st = static_ws_address(&ws);
    if (st != RET_OK) return st;
    // Nothing in the scratch needs to start at zero: the prep pass writes every
    // byte the tensor-core kernel reads.
    return launch_chunkwise_ws(a, ws, s);
}

}  // namespace ret
