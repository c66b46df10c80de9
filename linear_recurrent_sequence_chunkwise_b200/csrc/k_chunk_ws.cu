// k_chunk_ws.cu -- chunkwise retention forward with a caller-provided
// workspace: a bandwidth-bound prep kernel plus a warp-specialized
// tcgen05 / TMEM / TMA kernel.
//
// Same mathematics as k_chunk_tc.cu ("Hybrid Architectures: RetNet and the
// Three Computation Paradigms", section 7.2; RetNet paper summary, Eq. 7),
// with the decay folded into a scaled key k'_c = gamma^(L-1-c) k_c (c the row
// in its chunk of L rows), a pre-scaled state T = gamma^L R and a row scale:
//     out_r = gamma^(r+1-L) [ sum_{c<=r} (q_r . k'_c) v_c + q_r^T T ],
//     R     = T + K'^T V.
//
// 1. k_prep_qk (HBM-bound, one pass): rotates q and k once per head (xPos,
//    consecutive pairs, angle (pos_offset + n) theta_p with the sine and
//    cosine of each (position, pair) evaluated once for all heads), scales
//    each rotated key row by its zeta, and writes q_rot and k' (bf16) into the
//    workspace.  Without rotation only k' is written and q is read in place.
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
//                state:    R = gamma^L R + dS in registers (fp32), then the
//                          bf16 T = gamma^L' R into smem for the next read-out,
//                epilogue: out = gamma^(r+1-L) O staged in the chunk's V slot.
//    TMEM columns: A [0,128), P [128,192), O [192,256), Q [256,384),
//    dS [384,512).  Every hand-off between the roles has at least one block
//    of MMAs in between, so no role waits on another in the steady state.
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
                // zeta = gamma^(L-1-r): the exponent in fp64, exp2 in fp32 (relative error ~1e-7)
                const float zeta = exp2f((float)((double)(L - 1 - r) * hc.log2g[h0 + hh]));
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
};

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

template <int DK, typename Tout>
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
    const int h = ((int)blockIdx.x / nt) % p.H, b = (int)blockIdx.x / (nt * p.H);
    const int j0 = jt * kW;
    const int N = p.N;
    const int nchunks = (N + kC - 1) / kC;
    const double lg = p.hc.log2g[h];
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
                    tc::tma_load_4d(sm + WsSmem<DK>::kQ + s * (kC * 128), &p.tq, &bars.qfull, 64 * s, h, n0, b);
                for (int part = 0; part < kParts && ok; part++) {
                    const int g = jc * kParts + part, slot = g % kKSlots, u = g / kKSlots;
                    if (u > 0) ok = tc::mbar_wait(&bars.kempty[slot], (u - 1) & 1);
                    if (!ok) break;
                    uint8_t* dst = sm + WsSmem<DK>::kK + slot * kKPartBytes;
                    tc::mbar_arrive_expect_tx(&bars.kfull[slot], kKPartBytes);
                    for (int s = 0; s < 2; s++)
                        tc::tma_load_4d(dst + s * (kC * 128), &p.tk, &bars.kfull[slot], part * kPartDk + 64 * s, h,
                                        n0, b);
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
        // decay powers of a full chunk and of the (possibly shorter) last one
        const int L_last = N - (nchunks - 1) * kC;
        const float g_full = (float)exp2((double)kC * lg);
        const float sc_full = (float)exp2((double)(r + 1 - kC) * lg);
        const float g_last = (float)exp2((double)L_last * lg);
        const float sc_last = (float)exp2((double)(r + 1 - L_last) * lg);
        if (has_init) {
            // Continue from the given state: R = S_init, and the first read-out
            // uses T = gamma^L0 S_init (L0 the first chunk's length).
            const float g0 = nchunks == 1 ? g_last : g_full;
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
                const float gL = last ? g_last : g_full;
#pragma unroll
                for (int part = 0; part < kParts; part++) {
                    uint32_t d[32];
                    tc::tmem_ld32(tb + lane_off + kTD + part * kW + 32 * wg, d);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; i++) R[part][i] = fmaf(gL, R[part][i], __uint_as_float(d[i]));
                }
                tc::tc_fence_before();
                elect_arrive(&bars.dsfree, lane);
                if (!last) {
                    const float gN = (jc + 1 == nchunks - 1) ? g_last : g_full;
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
                        const float sc = (last ? sc_last : sc_full) * rs;
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
                            const float sc = (last ? sc_last : sc_full) * rs;
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
                    const float sc = (last ? sc_last : sc_full) * rs;
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
    auto kern = k_chunkwise_ws<DK, Tout>;
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

bool chunkwise_ws_supported(const RetArgs& a) {
    if (a.in_dt != RET_BF16) return false;
    if (a.chunk != kC || !(a.dk == 128 || a.dk == 256) || a.dv % kW != 0) return false;
    if (a.N > (1 << 30)) return false;
    if ((long long)a.B * a.H * (a.dv / kW) > (1ll << 30)) return false;
    for (int h = 0; h < a.H; h++)
        if (!(a.hc.log2g[h] * kC >= -60.0)) return false;
    return true;
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
