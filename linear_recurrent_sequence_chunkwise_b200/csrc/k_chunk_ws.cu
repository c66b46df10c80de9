// k_chunk_ws.cu -- chunkwise retention forward on the tensor cores: a
// warp-specialized tcgen05 / TMEM / TMA kernel fed by a pass that rotates q
// and k and scales the keys (and, in the scores form, also computes the
// masked intra-chunk scores P on the tensor cores).
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
// Two forms share the main kernel.  The scores form (the allocating call,
// the workspace call, prepare/prepared and the normalised forward) runs
// k_prep_scores (below, after the main kernel) and then k_chunkwise_ws with
// PREP = true: the scores P = tril(Q K'^T) of each (batch, head, chunk) come
// from the workspace, warp 1 issues only the read-out and P V (P as the
// shared-memory A operand, loaded by the producer), and the transform
// warpgroups skip the mask.  The two-pass form (the backward's passes, the
// MSR layer, the allocation-free call) runs k_prep_qk and then
// k_chunkwise_ws with PREP = false, as laid out here:
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
//                slow the tensor pipe down);
//      warps 8-15 (two warpgroups on TMEM lanes 0..127, one column half each):
//                mask:     P = tril(A) -> packed bf16 in TMEM,
//                state:    R = gamma^L R + gamma^(L-1-a) dS in registers
//                          (fp32), then the bf16 T = gamma^(a'+1) R into smem
//                          for the next read-out,
//                epilogue: out = gamma^(r-a) O staged in the chunk's V slot.
//    TMEM columns: A [0,128), P [128,192), O [192,256), Q [256,384),
//    dS [384,512) (the scores form leaves A and P unused).  Every hand-off
//    between the roles has at least one block of MMAs in between, so no role
//    waits on another in the steady state.  On B200 the kernel is bound by
//    its SM's shared-memory port (TMA fills, tensor-core operand reads and
//    the warps' staging traffic, about 560 KB a chunk in the scores form).
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
    // PREP instances: the masked scores P of every (b, h, chunk), bf16
    // [B, H, nchunks, 128 query rows, 128 key columns]: tile rows
    // ((b H + h) nchunks + j) 128 of a 2-D map {128, rows}.
    CUtensorMap tp;
};

constexpr int kKSlots = 3;                         // K' ring depth (parts of 128 d_k rows)
constexpr int kKPartBytes = kPartDk * kC * 2;      // 32 KB

constexpr int kPBytes = kC * kC * 2;              // 32 KB: the masked scores P of one chunk (bf16)

// With precomputed scores (PREP) the K' parts are read by the state-update
// issuer alone, so their ring takes two slots and the third one's space
// holds the chunk's P tile.
template <int DK, bool PREP>
struct WsSmem {
    static constexpr int kSlots = PREP ? 2 : kKSlots;
    static constexpr uint32_t kQ = 0;                              // Q staging, DK x 128 rows
    static constexpr uint32_t kK = kQ + DK * kC * 2;               // K' ring
    static constexpr uint32_t kP = kK + kSlots * kKPartBytes;      // P tile (PREP)
    static constexpr uint32_t kV = kP + (PREP ? kPBytes : 0);      // 2 x 16 KB
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
    uint64_t pfull, pempty;   // the P tile's slot (precomputed scores)
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

template <int DK, typename Tout, bool PREP>
__global__ void __launch_bounds__(kThreads, 1) k_chunkwise_ws(const __grid_constant__ WsParams p) {
    using Sm = WsSmem<DK, PREP>;
    constexpr int kSl = Sm::kSlots;   // K' ring slots
    constexpr int kParts = DK / kPartDk;
    constexpr int kQSlabs = DK / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ Bars bars;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = p.dv / kW, jt = (int)blockIdx.x % nt;     // this CTA's 64 value columns
    const int h = ((int)blockIdx.x / nt) % p.H, b = (int)blockIdx.x / (nt * p.H);
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
        for (int i = 0; i < kSl; i++) {
            tc::mbar_init(&bars.kfull[i], 1);
            tc::mbar_init(&bars.kempty[i], PREP ? 1 : 2);  // read by both issuers (one with P given)
        }
        tc::mbar_init(&bars.pfull, 1);
        tc::mbar_init(&bars.pempty, 1);
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
        if (PREP) tc::prefetch_tmap(&p.tp);
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
            // (the CTAs of a head split the Q and K' boxes between them)
            auto prefetch = [&](int jp) {
                if (jp >= nchunks) return;
                const int n0p = jp * kC;
                for (int i = jt; i < 2 * kQSlabs; i += nt)
                    tc::tma_prefetch_l2_4d(i < kQSlabs ? &p.tq : &p.tk, 64 * (i % kQSlabs), h, n0p, b);
                tc::tma_prefetch_l2_4d(&p.tv, j0, h, n0p, b);
            };
            prefetch(0);
            prefetch(1);
            for (int jc = 0; jc < nchunks && ok; jc++) {
                const int n0 = jc * kC;
                prefetch(jc + 2);
                if (jc > 0) ok = tc::mbar_wait(&bars.qempty, (jc - 1) & 1);
                if (!ok) break;
                tc::mbar_arrive_expect_tx(&bars.qfull, DK * kC * 2);
                for (int s = 0; s < kQSlabs; s++)
                    tc::tma_load_4d(sm + Sm::kQ + s * (kC * 128), &p.tq, &bars.qfull, 64 * s, h, n0, b);
                for (int part = 0; part < kParts && ok; part++) {
                    const int g = jc * kParts + part, slot = g % kSl, u = g / kSl;
                    if (u > 0) ok = tc::mbar_wait(&bars.kempty[slot], (u - 1) & 1);
                    if (!ok) break;
                    uint8_t* dst = sm + Sm::kK + slot * kKPartBytes;
                    tc::mbar_arrive_expect_tx(&bars.kfull[slot], kKPartBytes);
                    for (int s = 0; s < 2; s++)
                        tc::tma_load_4d(dst + s * (kC * 128), &p.tk, &bars.kfull[slot], part * kPartDk + 64 * s, h,
                                        n0, b);
                }
                const int vs = jc & 1;
                if (ok && jc >= 2) ok = tc::mbar_wait(&bars.vempty[vs], ((jc >> 1) & 1) ^ 1);
                if (!ok) break;
                tc::mbar_arrive_expect_tx(&bars.vfull[vs], kVBytes);
                tc::tma_load_4d(sm + Sm::kV + vs * kVBytes, &p.tv, &bars.vfull[vs], j0, h, n0, b);
                if constexpr (PREP) {
                    // the chunk's masked scores, once the P V of the previous chunk is done
                    if (jc > 0) ok = tc::mbar_wait(&bars.pempty, (jc - 1) & 1);
                    if (!ok) break;
                    const int prow = ((b * p.H + h) * nchunks + jc) * kC;
                    tc::mbar_arrive_expect_tx(&bars.pfull, kPBytes);
                    for (int s = 0; s < 2; s++)
                        tc::tma_load_2d(sm + Sm::kP + s * (kC * 128), &p.tp, &bars.pfull, 64 * s, prow);
                }
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
                    uint8_t* slot = sm + Sm::kV + vs * kVBytes;
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
            const uint64_t dk_mn = tc::sdesc_sw128(tc::smem_u32(sm + Sm::kK), kC * 128, 1024);
            const uint64_t dv_mn = tc::sdesc_sw128(tc::smem_u32(sm + Sm::kV), kC * 128, 1024);
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
                    const int g = jc * kParts + part, slot = g % kSl, u = g / kSl;
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
            const uint64_t dk_k = tc::sdesc_sw128(tc::smem_u32(sm + Sm::kK), 16, 1024);         // K' as B, K-major
            const uint64_t dv_mn = tc::sdesc_sw128(tc::smem_u32(sm + Sm::kV), kC * 128, 1024);  // V as B, MN-major
            const uint64_t dt_mn = tc::sdesc_sw128(tc::smem_u32(sm + Sm::kT), DK * 128, 1024);  // T as B, MN-major
            // a timed-out wait must leave the warp converged for elect.sync
            auto wait = [&](uint64_t* bar, uint32_t parity) {
                return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity));
            };
            // Per chunk: A = Q K'^T part by part with dS = K'^T V of every part
            // but the last right behind it (so each K' part is released early),
            // then the read-out O = Q T, the last dS part, and O += P V.
            // With precomputed scores: the read-out, then O += P V with P as the
            // shared-memory A operand (K-major, 128-byte swizzle).
            const uint64_t dp_k = tc::sdesc_sw128(tc::smem_u32(sm + Sm::kP), 16, 1024);
            for (int jc = 0; PREP && jc < nchunks && ok; jc++) {
                const uint32_t vo = (uint32_t)((jc & 1) * kVBytes) >> 4;
                ok = wait(&bars.qready, jc & 1);
                if (!ok) break;
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
                ok = wait(&bars.pfull, jc & 1);
                if (ok) ok = wait(&bars.vfull[jc & 1], (jc >> 1) & 1);
                if (!ok) break;
                tc::tc_fence_after();
#pragma unroll
                for (int k = 0; k < kC / 16; k++)
                    tc::mma_bf16_ss_elect(tb + kTO, dp_k + (uint32_t)(((k / 4) * (kC * 128) + (k % 4) * 32) >> 4),
                                          dv_mn + vo + (uint32_t)((k * 2048) >> 4), id_pv,
                                          (jc > 0) || has_init || (k > 0));
                tc::mma_commit_elect(&bars.ofull);
                tc::mma_commit_elect(&bars.pempty);
                if (!p.tma_out) tc::mma_commit_elect(&bars.vempty[jc & 1]);
            }
            for (int jc = 0; !PREP && jc < nchunks && ok; jc++) {
                const uint32_t vo = (uint32_t)((jc & 1) * kVBytes) >> 4;
                ok = wait(&bars.qready, jc & 1);
                if (ok && jc > 0) ok = wait(&bars.aread, (jc - 1) & 1);
                if (!ok) break;
                for (int part = 0; part < kParts && ok; part++) {
                    const int g = jc * kParts + part, slot = g % kSl, u = g / kSl;
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
        const uint8_t* sQ = sm + Sm::kQ;
        uint4 qv[DK / 8];
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
        uint8_t* sT = sm + Sm::kT;
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
            // (with precomputed scores there is no mask step)
            if (!PREP) ok = tc::mbar_wait(&bars.afull, jc & 1);
            if (!ok) break;
            tc::tc_fence_after();
            if (!PREP) {
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
                tc::tc_fence_before();
                elect_arrive(&bars.pready, lane);
            }
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
                        uint8_t* sO = sm + Sm::kV + (jc & 1) * kVBytes;
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
                            uint8_t* sO = sm + Sm::kV + (jc & 1) * kVBytes;
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

// ------------------------------------------------------------ scores pass
//
// k_prep_scores: persistent and warp-specialized; each CTA walks the tiles
// (batch, head, chunk) blockIdx.x, blockIdx.x + gridDim.x, ..., one 64-column
// slab of d_k at a time through a ring of kScStages shared-memory stages:
//   warp 0 (one lane)   TMA: the slab of the chunk's raw q and k rows into a
//                       stage (128-byte swizzle; a d_k below DK reads as
//                       zeros past its end, and so do rows past the sequence);
//   warps 4-7           turn each consecutive pair in place (xPos, angle
//                       (pos_offset + n) theta_p: a thread's first row from the
//                       position, fp64 angle reduced, fp32 sine and cosine; its
//                       next rows by turning through the row step), scale each
//                       key row by gamma^(a-r), and store the slab of q_rot
//                       (when copied) and of k' to the workspace by TMA;
//   warp 1 (one lane)   tcgen05: A' += Q_slab K'_slab^T (M = N = 128, K = 64,
//                       both operands from the stage) into one of two TMEM
//                       accumulators;
//   warps 8-11          P = tril(A') -> bf16 in the 128-byte swizzle of the
//                       K-major A operand the main kernel's P V reads, staged
//                       and stored by TMA.
// A stage is free once its MMAs are done and its stores have read it; an
// accumulator once the previous tile's P has been read out of it.  Every wait
// is bounded; a warpgroup agrees on each wait's outcome (named barriers 1
// and 2), and a timed-out wait ends the CTA's walk with the error word set.
struct ScoreParams {
    CUtensorMap tq_in, tk_in;      // raw q, k: {dk, H, N, B}, row pitch q_ld / k_ld
    CUtensorMap tq_out, tk_out;    // q_rot, k' in the workspace: {DK, H, N, B}
    CUtensorMap tp;                // P tiles: {128, B H nchunks 128}
    HeadConsts hc;
    int N, H, nchunks, ntiles, dks, xpos, qcopy;
    long long pos0;
    double theta[128];             // theta_p = base^(-2p/d_k) of every pair, fp64
};

constexpr int kScThreads = 512;
constexpr int kScStages = 5;
constexpr int kScLag = 2;                        // slabs whose stores may still be reading their stages
constexpr uint32_t kScSlab = kC * 128;           // one 64-column slab of 128 rows: 16 KB
constexpr uint32_t kScStage = 2 * kScSlab;       // q and k slabs

// The rotation's tables (fp32 cosine, sine pairs): rows 0..15 the turn
// through r theta_p, row 16 through 16 theta_p (a thread's row step), row 17
// the current tile's base angle (pos_offset + n0) theta_p.
constexpr int kScTabRows = 18;

struct ScSmem {
    static constexpr uint32_t kRing = 0;
    static constexpr uint32_t kP = kRing + kScStages * kScStage;
    static constexpr uint32_t kTab = kP + kPBytes;
    static constexpr uint32_t kEnd = kTab + kScTabRows * 128 * 8;
    static constexpr uint32_t kBytes = kEnd + 1024;
};

struct ScBars {
    uint64_t full[kScStages], empty[kScStages], rotated[kScStages], accfull[2], accempty[2];
};

// Named barrier `id` over n threads (128 unless given), returning whether x
// holds in all of them.
__device__ __forceinline__ bool wg_all_id(int id, bool x, int n = 128) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)x), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

template <int DK>
__global__ void __launch_bounds__(kScThreads, 1) k_prep_scores(const __grid_constant__ ScoreParams p) {
    // the slabs of d_k a tile has: a d_k below DK (zero-padded) skips the
    // slabs past it, which the main kernel reads as TMA zero-fill
    const int nslabs = (p.dks + 63) / 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ ScBars bars;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the tile of local index i: (bh, jc), the (batch, head) pairs of one chunk
    // next to each other, so that the CTAs at work read whole token rows of q
    // and k together; heads the tensor cores do not take are skipped
    const int BH = p.ntiles / p.nchunks;
    auto tile_of = [&](int i, int* bh, int* jc) {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        *jc = t / BH;
        *bh = t % BH;
    };
    const int ntile = p.ntiles > (int)blockIdx.x ? (p.ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int i = 0; i < kScStages; i++) {
            tc::mbar_init(&bars.full[i], 1);
            tc::mbar_init(&bars.empty[i], 2);     // the MMAs and the stores have read it
            tc::mbar_init(&bars.rotated[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&bars.accfull[i], 1);
            tc::mbar_init(&bars.accempty[i], 4);  // the epilogue warps have read it
        }
        s_fail = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(&s_tmem, 256);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tb = s_tmem;
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            int done = 0;   // tiles loaded (the stages run over their slabs in order)
            for (int i = 0; i < ntile && ok; i++) {
                int bh, jc;
                tile_of(i, &bh, &jc);
                const int h = bh % p.H, b = bh / p.H;
                if (p.hc.anchor[h] < 0) continue;
                for (int s = 0; s < nslabs && ok; s++) {
                    const int g = done * nslabs + s, st = g % kScStages, u = g / kScStages;
                    if (u > 0) ok = tc::mbar_wait(&bars.empty[st], (u - 1) & 1);
                    if (!ok) break;
                    uint8_t* dst = sm + ScSmem::kRing + st * kScStage;
                    tc::mbar_arrive_expect_tx(&bars.full[st], kScStage);
                    tc::tma_load_4d(dst, &p.tq_in, &bars.full[st], 64 * s, h, jc * kC, b);
                    tc::tma_load_4d(dst + kScSlab, &p.tk_in, &bars.full[st], 64 * s, h, jc * kC, b);
                }
                done++;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        const uint32_t id = tc::idesc_bf16_f32(128, 128, 0, 0);
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, tc::mbar_wait(bar, parity));
        };
        int done = 0;   // tiles issued (the accumulators alternate over them)
        for (int i = 0; i < ntile && ok; i++) {
            int bh, jc;
            tile_of(i, &bh, &jc);
            if (p.hc.anchor[bh % p.H] < 0) continue;
            const int buf = done & 1;
            if (done >= 2) ok = wait(&bars.accempty[buf], ((done >> 1) - 1) & 1);
            if (!ok) break;
            for (int s = 0; s < nslabs && ok; s++) {
                const int g = done * nslabs + s, st = g % kScStages, u = g / kScStages;
                ok = wait(&bars.rotated[st], u & 1);
                if (!ok) break;
                tc::tc_fence_after();
                const uint32_t base = tc::smem_u32(sm + ScSmem::kRing + st * kScStage);
                const uint64_t dq = tc::sdesc_sw128(base, 16, 1024);
                const uint64_t dk = tc::sdesc_sw128(base + kScSlab, 16, 1024);
#pragma unroll
                for (int k = 0; k < 4; k++)
                    tc::mma_bf16_ss_elect(tb + 128 * buf, dq + (uint32_t)(k * 2), dk + (uint32_t)(k * 2), id,
                                          (s > 0) || (k > 0));
                tc::mma_commit_elect(&bars.empty[st]);
            }
            if (!ok) break;
            tc::mma_commit_elect(&bars.accfull[buf]);
            done++;
        }
    } else if ((warp >= 4 && warp < 8) || warp >= 12) {
        // ------------------------------------------ rotation (two warpgroups)
        constexpr int kRot = 256;             // rotation threads
        const int wt = warp < 8 ? tid - 128 : tid - 256;   // 0..255
        const int c16 = wt % 8;               // the thread's 16-byte chunk of a slab row
        const int rfirst = wt / 8;            // rows rfirst, rfirst + 32, ...
        float2* tab = reinterpret_cast<float2*>(sm + ScSmem::kTab);   // [kScTabRows][128]
        const int npairs = p.dks / 2;
        if (p.xpos) {
            // turns through r theta_p, r = 0..16 (small angles: fp32 sine and cosine)
            for (int e = wt; e < 17 * 128; e += kRot) {
                const int r = e / 128, pp = e % 128;
                float sv = 0.f, cv = 1.f;
                if (pp < npairs) sincosf((float)(r * p.theta[pp]), &sv, &cv);
                tab[e] = make_float2(cv, sv);
            }
        }
        int done = 0;
        for (int i = 0; i < ntile && ok; i++) {
            int bh, jc;
            tile_of(i, &bh, &jc);
            const int h = bh % p.H, b = bh / p.H;
            if (p.hc.anchor[h] < 0) continue;
            const int n0 = jc * kC, L = min(kC, p.N - n0);
            const float lgf = (float)p.hc.log2g[h];
            const int a = min(p.hc.anchor[h], L - 1);
            if (p.xpos) {
                // the tile's base angle of every pair: fp64 product, reduced, then fp32
                if (wt < npairs) {
                    float sv, cv;
                    __sincosf(angle_mod_2pi((double)(p.pos0 + n0) * p.theta[wt]), &sv, &cv);
                    tab[17 * 128 + wt] = make_float2(cv, sv);
                }
                wg_all_id(1, true, kRot);
            }
            for (int s = 0; s < nslabs && ok; s++) {
                const int g = done * nslabs + s, st = g % kScStages, u = g / kScStages;
                ok = wg_all_id(1, tc::mbar_wait(&bars.full[st], u & 1), kRot);
                if (!ok) break;
                uint8_t* base = sm + ScSmem::kRing + st * kScStage;
                const int col = 64 * s + 8 * c16;   // first of the thread's 8 columns
                const bool real = col < p.dks;
                const bool turn = p.xpos && real;
                if (real) {
                    float cs[4], sn[4], cst[4], sst[4];
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        cs[k] = cst[k] = 1.f;
                        sn[k] = sst[k] = 0.f;
                        if (turn) {
                            const int pp = col / 2 + k;
                            const float2 t0 = tab[17 * 128 + pp], t2 = tab[16 * 128 + pp];
                            float2 t1 = tab[(rfirst & 15) * 128 + pp];
                            if (rfirst >= 16) t1 = make_float2(t1.x * t2.x - t1.y * t2.y, t1.y * t2.x + t1.x * t2.y);
                            cs[k] = t0.x * t1.x - t0.y * t1.y;   // turn through (pos0 + n0 + rfirst) theta_p
                            sn[k] = t0.y * t1.x + t0.x * t1.y;
                            cst[k] = t2.x * t2.x - t2.y * t2.y;  // the row step: 32 theta_p
                            sst[k] = 2.f * t2.x * t2.y;
                        }
                    }
                    // the thread's rows rfirst + 32 i, i < nr: every load first, then
                    // the turns and stores (two warps per sub-partition here, so the
                    // loads' latency is hidden mostly by the thread's own work)
                    const int nr = (L - rfirst + 31) >> 5;
                    uint4 qv[4], kv[4];
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        if (i < nr) {
                            const uint32_t off = tc::sw128_off((uint32_t)(rfirst + 32 * i), (uint32_t)c16);
                            if (turn) qv[i] = *reinterpret_cast<const uint4*>(base + off);
                            kv[i] = *reinterpret_cast<const uint4*>(base + kScSlab + off);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        if (i < nr) {
                            const int r = rfirst + 32 * i;
                            const uint32_t off = tc::sw128_off((uint32_t)r, (uint32_t)c16);
                            // k' scale gamma^(a-r) (fp32: relative error a few 1e-7)
                            const float zeta = exp2f((float)(a - r) * lgf);
                            float ck[4], sk[4];
#pragma unroll
                            for (int k = 0; k < 4; k++) {
                                ck[k] = cs[k] * zeta;
                                sk[k] = sn[k] * zeta;
                            }
                            if (turn) *reinterpret_cast<uint4*>(base + off) = turn_group(qv[i], cs, sn);
                            *reinterpret_cast<uint4*>(base + kScSlab + off) = turn_group(kv[i], ck, sk);
                            if (turn) {
#pragma unroll
                                for (int k = 0; k < 4; k++) {
                                    const float c2 = cs[k] * cst[k] - sn[k] * sst[k];
                                    sn[k] = sn[k] * cst[k] + cs[k] * sst[k];
                                    cs[k] = c2;
                                }
                            }
                        }
                    }
                }
                tc::fence_proxy_async_smem();
                wg_all_id(1, true, kRot);
                if (wt == 0) {
                    if (p.qcopy) tc::tma_store_4d(&p.tq_out, base, 64 * s, h, n0, b);
                    tc::tma_store_4d(&p.tk_out, base + kScSlab, 64 * s, h, n0, b);
                    tc::bulk_commit_group();
                    tc::mbar_arrive(&bars.rotated[st]);
                    // the stores of slab g - kScLag have read their stage by now
                    // (one bulk group per slab): that stage goes back
                    tc::bulk_wait_group_read<kScLag>();
                    if (g >= kScLag) tc::mbar_arrive(&bars.empty[(g - kScLag) % kScStages]);
                }
            }
            done++;
        }
        if (wt == 0) tc::bulk_wait_group<0>();   // (no load waits for the last stages)
    } else if (warp >= 8) {
        // ------------------------------------------- epilogue warpgroup (warps 8-11)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int wt = tid - 256;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        int done = 0;
        for (int i = 0; i < ntile && ok; i++) {
            int bh, jc;
            tile_of(i, &bh, &jc);
            if (p.hc.anchor[bh % p.H] < 0) continue;
            const int buf = done & 1;
            ok = wg_all_id(2, tc::mbar_wait(&bars.accfull[buf], (done >> 1) & 1));
            if (!ok) break;
            tc::tc_fence_after();
            // the staging tile is reused once the previous P store has read it
            if (wt == 0) tc::bulk_wait_group_read<0>();
            wg_all_id(2, true);
#pragma unroll
            for (int q32 = 0; q32 < 4; q32++) {
                uint32_t av[32], w[16];
                tc::tmem_ld32(tb + lane_off + 128 * buf + 32 * q32, av);
                tc::tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; k++) {
                    const int c = 32 * q32 + 2 * k;
                    const float lo = (c <= r) ? __uint_as_float(av[2 * k]) : 0.f;
                    const float hi = (c + 1 <= r) ? __uint_as_float(av[2 * k + 1]) : 0.f;
                    w[k] = tc::pack_bf16x2(lo, hi);
                }
                // columns 32 q32 .. + 31: slab q32 / 2, 16-byte chunks 4 (q32 % 2) ..
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++)
                    *reinterpret_cast<uint4*>(sm + ScSmem::kP + (q32 / 2) * kScSlab +
                                              tc::sw128_off((uint32_t)r, (uint32_t)(4 * (q32 % 2) + q4))) =
                        make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
            }
            tc::tc_fence_before();
            elect_arrive(&bars.accempty[buf], lane);
            tc::fence_proxy_async_smem();
            wg_all_id(2, true);
            if (wt == 0) {
                const int prow = (bh * p.nchunks + jc) * kC;
                for (int s = 0; s < 2; s++) tc::tma_store_2d(&p.tp, sm + ScSmem::kP + s * kScSlab, 64 * s, prow);
                tc::bulk_commit_group();
            }
            done++;
        }
        if (wt == 0) tc::bulk_wait_group<0>();
    }
    if (!ok) atomicExch(&s_fail, 1);
    tc::tc_fence_before();
    __syncthreads();
    if (s_fail && tid == 0) atomicExch(&g_err_chunk_ws, kErrTimeout);
    if (warp == 1) tc::tmem_dealloc(tb, 256);
}

template <int DK, typename Tout, bool PREP = false>
ret_status launch_main(const WsParams& p, cudaStream_t s) {
    auto kern = k_chunkwise_ws<DK, Tout, PREP>;
    const int smem = (int)WsSmem<DK, PREP>::kBytes;
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
    // a d_k padded to the kernel's: the padded columns are read as TMA
    // zero-fill, so the workspace need not hold them
    const uint64_t dq[4] = {(uint64_t)(a.dk_real ? a.dk_real : a.dk), H, N, B};
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

// ------------------------------------------------------- the scores form

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static int chunks_of(const RetArgs& a) { return (a.N + kC - 1) / kC; }

// Workspace of the scores form: that of the two-pass form (k', then q_rot),
// then the P tiles [B, H, nchunks, 128, 128] bf16.
size_t chunkwise_scores_bytes(const RetArgs& a) {
    return align256(chunkwise_ws_bytes(a)) + (size_t)a.B * a.H * chunks_of(a) * kPBytes;
}

// The P tiles' tensor map (both passes use the same one).
static bool scores_map(const RetArgs& a, void* ws, CUtensorMap* tp) {
    void* pbuf = reinterpret_cast<uint8_t*>(ws) + align256(chunkwise_ws_bytes(a));
    const uint64_t prows = (uint64_t)a.B * a.H * chunks_of(a) * kC;
    const uint64_t dpp[2] = {(uint64_t)kC, prows};
    const uint64_t spp[1] = {(uint64_t)kC * 2};
    const uint32_t bpp[2] = {64, (uint32_t)kC};
    return make_tmap_bf16(tp, pbuf, 2, dpp, spp, bpp, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Pass 1: rotation, key scale and the masked scores into the workspace.
ret_status launch_chunkwise_scores_pass1(const RetArgs& a, void* ws, cudaStream_t s) {
    __nv_bfloat16 *k_out, *q_rot;
    ws_parts(a, ws, &k_out, &q_rot);
    const bool qc = q_copied(a);
    const int nchunks = chunks_of(a);
    {
        ScoreParams sp;
        memset(&sp, 0, sizeof(sp));
        const int dkr = a.dk_real ? a.dk_real : a.dk;
        const uint64_t B = a.B, N = a.N, H = a.H, dk = a.dk;
        const uint64_t qld = a.q_ld ? a.q_ld : dkr, kld = a.k_ld ? a.k_ld : dkr;
        const uint32_t box[4] = {64, 1, (uint32_t)kC, 1};
        const uint64_t dr[4] = {(uint64_t)dkr, H, N, B};
        const uint64_t sq[3] = {qld * 2, H * qld * 2, N * H * qld * 2};
        const uint64_t sk[3] = {kld * 2, H * kld * 2, N * H * kld * 2};
        const uint64_t dw[4] = {dk, H, N, B};
        const uint64_t sw[3] = {dk * 2, H * dk * 2, N * H * dk * 2};
        if (!make_tmap_bf16(&sp.tq_in, a.q, 4, dr, sq, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_bf16(&sp.tk_in, a.k, 4, dr, sk, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_bf16(&sp.tk_out, k_out, 4, dw, sw, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            (qc && !make_tmap_bf16(&sp.tq_out, q_rot, 4, dw, sw, box, CU_TENSOR_MAP_SWIZZLE_128B)) ||
            !scores_map(a, ws, &sp.tp))
            return RET_ERR_CUDA;
        sp.hc = a.hc;
        sp.N = a.N;
        sp.H = a.H;
        sp.nchunks = nchunks;
        sp.dks = dkr;
        sp.xpos = a.xpos;
        sp.qcopy = qc ? 1 : 0;
        sp.pos0 = a.pos_offset;
        for (int i = 0; i < 128; i++) sp.theta[i] = i < dkr / 2 ? pow(a.theta_base, -2.0 * i / dkr) : 0.0;
        const long long ntiles = (long long)a.B * a.H * nchunks;
        if (ntiles > (1ll << 30)) return fail(RET_ERR_UNSUPPORTED, "chunkwise (scores): too many chunks");
        sp.ntiles = (int)ntiles;
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                      cudaSuccess)
            return fail(RET_ERR_CUDA, "chunkwise (scores pass): device query failed");
        const unsigned grid = (unsigned)std::min<long long>(ntiles, sms);
        const int smem = (int)ScSmem::kBytes;
        if (a.dk == 256) {
            auto kern = k_prep_scores<256>;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
                return check_launch("chunkwise (scores pass): smem attribute");
            kern<<<grid, kScThreads, smem, s>>>(sp);
        } else {
            auto kern = k_prep_scores<128>;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
                return check_launch("chunkwise (scores pass): smem attribute");
            kern<<<grid, kScThreads, smem, s>>>(sp);
        }
        return check_launch("chunkwise (scores pass)");
    }
}

// Pass 2: read-out, P V and state update on the prepared rows and scores
// (a.initial_state honoured).
ret_status launch_chunkwise_scores_pass2(const RetArgs& a, void* ws, cudaStream_t s) {
    __nv_bfloat16 *k_out, *q_rot;
    ws_parts(a, ws, &k_out, &q_rot);
    const bool qc = q_copied(a);
    WsParams p;
    ret_status st = fill_params(&p, a, qc ? (const void*)q_rot : a.q, qc || !a.q_ld ? a.dk : a.q_ld, k_out);
    if (st != RET_OK) return st;
    if (!scores_map(a, ws, &p.tp)) return RET_ERR_CUDA;
    const bool f32 = a.out_dt == RET_F32;
    if (a.dk == 256) return f32 ? launch_main<256, float, true>(p, s) : launch_main<256, __nv_bfloat16, true>(p, s);
    return f32 ? launch_main<128, float, true>(p, s) : launch_main<128, __nv_bfloat16, true>(p, s);
}

ret_status launch_chunkwise_scores(const RetArgs& a, void* ws, cudaStream_t s) {
    const ret_status st = launch_chunkwise_scores_pass1(a, ws, s);
    return st != RET_OK ? st : launch_chunkwise_scores_pass2(a, ws, s);
}

// The scores form on scratch from a stream-ordered pool the library keeps per
// device (created on the first call, never trimmed): allocated and freed in
// stream order around the launches, so concurrent calls on other streams get
// their own scratch.
ret_status launch_chunkwise_scores_pooled(const RetArgs& a, cudaStream_t s) {
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
    e = cudaMallocFromPoolAsync(&scratch, chunkwise_scores_bytes(a), pool, s);
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "chunkwise: scratch: %s", cudaGetErrorString(e));
    const ret_status st = launch_chunkwise_scores(a, scratch, s);
    e = cudaFreeAsync(scratch, s);
    if (st != RET_OK) return st;
    if (e != cudaSuccess) return fail(RET_ERR_CUDA, "chunkwise: scratch release: %s", cudaGetErrorString(e));
    return RET_OK;
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
