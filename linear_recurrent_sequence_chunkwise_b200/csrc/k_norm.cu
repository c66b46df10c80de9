// k_norm.cu -- retention with the score normalizations 2 and 3
// ("Hybrid Architectures: RetNet and the Three Computation Paradigms",
// section 8.5; RetNet paper summary, "Retention Score Normalization"):
//   2. D~_nm = D_nm / sqrt(sum_{i<=n} D_ni)
//   3. R~_nm = R_nm / max(|sum_{i<=n} R_ni|, 1),   R = (Q K^T) (.) D~
// Both divide row n of the score matrix by a scalar, so they scale output
// row n by f_n = c_n / max(|c_n s_n|, 1), with c_n = 1 / sqrt(sum_{i<=n}
// gamma^(n-i)) (a geometric series in closed form) and s_n = sum_{m<=n}
// gamma^(n-m) q_n . k_m = q_n . z_n, where z_n = gamma z_{n-1} + k_n is the
// decayed key sum: a recurrent d_k vector beside the state S, so the
// normalized retention keeps its chunkwise and recurrent forms.  The state S
// itself is unchanged.
//
// Chunkwise: three bandwidth-bound passes over the prepared q and k' (the
// keys already scaled by zeta = gamma^(L-1-c) within their chunk) fill a
// factor per (token, head) that the tensor-core kernel's epilogue applies:
//   k_keysum     sum of k' over each 32-row block,
//   k_keycarry   z before every chunk: z_j = gamma^L z_{j-1} + sum_c k'_c,
//   k_rowscale   s_n = gamma^(r+1-L) q_n . sum_{c<=r} k'_c + gamma^(r+1) q_n . z_{j-1}
//                for row r of chunk j, then f_n.
#include <cstring>

#include "kernels.h"

namespace ret {

namespace {

constexpr int kSub = 32;    // rows per key-sum block
constexpr int kChunk = 128;  // the workspace path's chunk

__device__ __forceinline__ void add_bf16x8(const uint4& u, float* acc) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 f = __bfloat1622float2(h[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
    }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* x) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 f = __bfloat1622float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

// One warp per (batch, head, 32-row block); lane g sums elements 8g..8g+7.
template <int DK>
__global__ void __launch_bounds__(256) k_keysum(const __nv_bfloat16* __restrict__ kp, float* __restrict__ subsum,
                                                int B, int N, int H, int nsub) {
    const int lane = threadIdx.x & 31;
    const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // (b * H + h) * nsub + s
    if (w >= (long long)B * H * nsub) return;
    const int s = (int)(w % nsub);
    const int bh = (int)(w / nsub), h = bh % H, b = bh / H;
    const int n0 = s * kSub, n1 = min(N, n0 + kSub);
    for (int g = lane; g < DK / 8; g += 32) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int n = n0; n < n1; n += 8) {
            uint4 x[8];
#pragma unroll
            for (int u = 0; u < 8; u++)
                if (n + u < n1)
                    x[u] = __ldg(reinterpret_cast<const uint4*>(kp + (((size_t)b * N + n + u) * H + h) * DK + 8 * g));
#pragma unroll
            for (int u = 0; u < 8; u++)
                if (n + u < n1) add_bf16x8(x[u], acc);
        }
        float4* dst = reinterpret_cast<float4*>(subsum + (size_t)w * DK + 8 * g);
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

// The decayed key sum before each chunk (zstart) and after the last one
// (z1).  Block (batch, head, 32 key components), thread (segment t,
// component): the chunks are cut into kSeg segments; each thread carries
// its segment from zero, the segments' end values are combined in order
// through shared memory (every segment before the last non-empty one spans
// `per` full chunks, so one decay factor serves them all), and each thread
// carries its segment again from its true start.
constexpr int kSeg = 8, kCarryD = 32;
__global__ void __launch_bounds__(kSeg * kCarryD) k_keycarry(const float* __restrict__ subsum, const float* z0,
                                                             float* zstart, float* z1, HeadConsts hc, int H, int DK,
                                                             int N, int nsub, int nch) {
    __shared__ float s_end[kSeg][kCarryD];
    const int slices = DK / kCarryD;
    const int bh = blockIdx.x / slices, h = bh % H;
    const int c = threadIdx.x % kCarryD, t = threadIdx.x / kCarryD;
    const int d = (blockIdx.x % slices) * kCarryD + c;
    const double lg = hc.log2g[h];
    const float g_full = (float)exp2(kChunk * lg);
    const float g_last = (float)exp2((N - (nch - 1) * kChunk) * lg);
    const int per = (nch + kSeg - 1) / kSeg, j0 = t * per, j1 = min(nch, j0 + per);
    const float g_seg = (float)exp2((double)per * kChunk * lg);  // decay over a full segment
    const float* ss = subsum + (size_t)bh * nsub * DK + d;
    constexpr int kPer = kChunk / kSub;
    auto chunk_sum = [&](int j) {
        float cs = 0.f;
#pragma unroll
        for (int i = 0; i < kPer; i++) {
            const int sb = j * kPer + i;
            if (sb < nsub) cs += ss[(size_t)sb * DK];
        }
        return cs;
    };
    // read before anything is written: z1 may be the same buffer as z0
    float Z = z0 ? z0[(size_t)bh * DK + d] : 0.f;
    // the segment's chunk sums, loaded together (segments of up to kHeld
    // chunks stay in registers for the second pass)
    constexpr int kHeld = 8;
    const bool held = j1 - j0 <= kHeld;
    float cs[kHeld];
#pragma unroll
    for (int u = 0; u < kHeld; u++) cs[u] = (held && j0 + u < j1) ? chunk_sum(j0 + u) : 0.f;
    auto sum_at = [&](int j) {
        if (held) {
            float v = 0.f;
#pragma unroll
            for (int u = 0; u < kHeld; u++) v = (j - j0 == u) ? cs[u] : v;
            return v;
        }
        return chunk_sum(j);
    };
    // pass 1: this segment from zero
    float E = 0.f;
    for (int j = j0; j < j1; j++) E = fmaf(j == nch - 1 ? g_last : g_full, E, sum_at(j));
    s_end[t][c] = E;
    __syncthreads();
    // the value entering this segment: the earlier (full) segments in order
    for (int u = 0; u < t; u++) Z = fmaf(g_seg, Z, s_end[u][c]);
    // pass 2: this segment from its true start
    for (int j = j0; j < j1; j++) {
        zstart[((size_t)bh * nch + j) * DK + d] = Z;
        Z = fmaf(j == nch - 1 ? g_last : g_full, Z, sum_at(j));
    }
    __syncthreads();  // every thread has read z0
    if (z1 && j1 == nch && j0 < j1) z1[(size_t)bh * DK + d] = Z;
}

// One warp per (batch, head, 32-row block): the row sums s_n of its rows and
// the factors f_n.  For row r of chunk j,
//   s = gamma^(r+1-L) q . P_r + gamma^(r+1) q . z_{j-1},  P_r = sum_{c<=r} k'_c,
// so each lane accumulates the two dot products over its 8 components, the
// lanes' partials are summed per row through shared memory, and the decay
// factors are applied once per row.
constexpr int kRsWarps = 4;  // warps per block of k_rowscale
template <int DK>
__global__ void __launch_bounds__(kRsWarps * 32, 6) k_rowscale(const __nv_bfloat16* __restrict__ qe,
                                                               const __nv_bfloat16* __restrict__ kp,
                                                               const float* __restrict__ subsum,
                                                               const float* __restrict__ zstart,
                                                               float* __restrict__ rowscale, HeadConsts hc, int B,
                                                               int N, int H, int nsub, int nch, long long pos0,
                                                               int flags) {
    static_assert(DK / 8 <= 32, "one 8-element group per lane");
    const int lane = threadIdx.x & 31;
    const long long w = (long long)blockIdx.x * kRsWarps + (threadIdx.x >> 5);
    if (w >= (long long)B * H * nsub) return;
    const int s = (int)(w % nsub);
    const int bh = (int)(w / nsub), h = bh % H, b = bh / H;
    const int j = s / (kChunk / kSub), n0c = j * kChunk, L = min(kChunk, N - n0c);
    const int r0 = (s % (kChunk / kSub)) * kSub;  // first row of the block within its chunk
    const int nrows = min(kSub, N - (n0c + r0));
    const bool act = (flags & kNormScore) && lane < DK / 8;  // without it only c_n is needed
    const double lg = hc.log2g[h];

    __shared__ float part[2][kRsWarps][kSub][33];  // (q . P, q . z) per row and lane
    float (*pp)[33] = part[0][threadIdx.x >> 5];
    float (*pz)[33] = part[1][threadIdx.x >> 5];
    if (flags & kNormScore) {
        float Z[8], P[8];
#pragma unroll
        for (int e = 0; e < 8; e++) Z[e] = P[e] = 0.f;
        if (act) {
            const float4* zs = reinterpret_cast<const float4*>(zstart + ((size_t)bh * nch + j) * DK + 8 * lane);
            const float4 z0 = zs[0], z1 = zs[1];
            Z[0] = z0.x; Z[1] = z0.y; Z[2] = z0.z; Z[3] = z0.w; Z[4] = z1.x; Z[5] = z1.y; Z[6] = z1.z; Z[7] = z1.w;
            for (int s2 = j * (kChunk / kSub); s2 < s; s2++) {
                const float4* ps = reinterpret_cast<const float4*>(subsum + ((size_t)bh * nsub + s2) * DK + 8 * lane);
                const float4 a0 = ps[0], a1 = ps[1];
                P[0] += a0.x; P[1] += a0.y; P[2] += a0.z; P[3] += a0.w;
                P[4] += a1.x; P[5] += a1.y; P[6] += a1.z; P[7] += a1.w;
            }
        }
#pragma unroll
        for (int rb = 0; rb < kSub; rb += 4) {
            uint4 kx[4], qx[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {
                if (act && rb + u < nrows) {
                    const size_t row = ((size_t)b * N + n0c + r0 + rb + u) * H + h;
                    kx[u] = __ldg(reinterpret_cast<const uint4*>(kp + row * DK + 8 * lane));
                    qx[u] = __ldg(reinterpret_cast<const uint4*>(qe + row * DK + 8 * lane));
                }
            }
#pragma unroll
            for (int u = 0; u < 4; u++) {
                float dP = 0.f, dZ = 0.f;
                if (act && rb + u < nrows) {
                    float kf[8], qf[8];
                    unpack_bf16x8(kx[u], kf);
                    unpack_bf16x8(qx[u], qf);
#pragma unroll
                    for (int e = 0; e < 8; e++) {
                        P[e] += kf[e];
                        dP = fmaf(qf[e], P[e], dP);
                        dZ = fmaf(qf[e], Z[e], dZ);
                    }
                }
                pp[rb + u][lane] = dP;
                pz[rb + u][lane] = dZ;
            }
        }
        __syncwarp();
    }
    if (lane < nrows) {
        const int r = r0 + lane;
        float sn = 0.f;
        if (flags & kNormScore) {
            float sP = 0.f, sZ = 0.f;
#pragma unroll 8
            for (int i = 0; i < 32; i++) {
                sP += pp[lane][i];
                sZ += pz[lane][i];
            }
            sn = exp2f((float)((r + 1 - L) * lg)) * sP + exp2f((float)((r + 1) * lg)) * sZ;
        }
        const long long n = n0c + r;
        double f = 1.0;
        if (flags & kNormDecay) {
            // sum_{i<=n} gamma^(n-i) over the whole sequence, position pos0 + n
            const double ln_g = lg * 0.69314718055994530942;
            const double cnt = (double)(pos0 + n + 1);
            const double geo = (lg == 0.0) ? cnt : expm1(cnt * ln_g) / expm1(ln_g);
            f = 1.0 / sqrt(geo);
        }
        if (flags & kNormScore) f /= fmax(fabs(f * (double)sn), 1.0);
        rowscale[((size_t)b * N + n) * H + h] = (float)f;
    }
}

struct NormLayout {
    size_t rowscale, subsum, zstart, total;
    int nsub, nch;
};

NormLayout norm_layout(const RetArgs& a) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    NormLayout L;
    L.nsub = (a.N + kSub - 1) / kSub;
    L.nch = (a.N + kChunk - 1) / kChunk;
    size_t o = al(chunkwise_scores_bytes(a));   // the scores form's k', q_rot and P tiles
    L.rowscale = o; o += al((size_t)a.B * a.N * a.H * 4);
    L.subsum = o; o += al((size_t)a.B * a.H * L.nsub * a.dk * 4);
    L.zstart = o; o += al((size_t)a.B * a.H * L.nch * a.dk * 4);
    L.total = o;
    return L;
}

}  // namespace

size_t normalized_ws_bytes(const RetArgs& a) { return norm_layout(a).total; }

ret_status launch_chunkwise_normalized(const RetArgs& a0, int flags, const float* z0, float* z1, void* ws,
                                       cudaStream_t s) {
    const NormLayout L = norm_layout(a0);
    uint8_t* base = reinterpret_cast<uint8_t*>(ws);
    float* rowscale = reinterpret_cast<float*>(base + L.rowscale);
    float* subsum = reinterpret_cast<float*>(base + L.subsum);
    float* zstart = reinterpret_cast<float*>(base + L.zstart);
    // the scores pass: k' opens the workspace, the rotated q follows it (xpos)
    // or is q itself, then the P tiles (the row factors scale whole output
    // rows, so the scores need no change)
    ret_status st = launch_chunkwise_scores_pass1(a0, ws, s);
    if (st != RET_OK) return st;
    const size_t qk = (size_t)a0.B * a0.N * a0.H * a0.dk;
    const __nv_bfloat16* kp = reinterpret_cast<const __nv_bfloat16*>(ws);
    const __nv_bfloat16* qe = a0.xpos ? kp + qk : reinterpret_cast<const __nv_bfloat16*>(a0.q);
    const long long warps = (long long)a0.B * a0.H * L.nsub;
    const int blocks = (int)((warps + 7) / 8);
    const int rs_blocks = (int)((warps + kRsWarps - 1) / kRsWarps);
    const bool keys = (flags & kNormScore) || z1;  // the key sums are needed
    if (a0.dk == 256) {
        if (keys) {
            k_keysum<256><<<blocks, 256, 0, s>>>(kp, subsum, a0.B, a0.N, a0.H, L.nsub);
            k_keycarry<<<a0.B * a0.H * (256 / kCarryD), kSeg * kCarryD, 0, s>>>(subsum, z0, zstart, z1, a0.hc,
                                                                                a0.H, 256, a0.N, L.nsub, L.nch);
        }
        k_rowscale<256><<<rs_blocks, kRsWarps * 32, 0, s>>>(qe, kp, subsum, zstart, rowscale, a0.hc, a0.B, a0.N, a0.H, L.nsub,
                                               L.nch, a0.pos_offset, flags);
    } else {
        if (keys) {
            k_keysum<128><<<blocks, 256, 0, s>>>(kp, subsum, a0.B, a0.N, a0.H, L.nsub);
            k_keycarry<<<a0.B * a0.H * (128 / kCarryD), kSeg * kCarryD, 0, s>>>(subsum, z0, zstart, z1, a0.hc,
                                                                                a0.H, 128, a0.N, L.nsub, L.nch);
        }
        k_rowscale<128><<<rs_blocks, kRsWarps * 32, 0, s>>>(qe, kp, subsum, zstart, rowscale, a0.hc, a0.B, a0.N, a0.H, L.nsub,
                                               L.nch, a0.pos_offset, flags);
    }
    st = check_launch("chunkwise normalized: row factors");
    if (st != RET_OK) return st;
    RetArgs a = a0;
    a.rowscale = rowscale;
    return launch_chunkwise_scores_pass2(a, ws, s);
}

}  // namespace ret
