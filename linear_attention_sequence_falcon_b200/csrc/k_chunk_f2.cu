// k_chunk_f2.cu -- chunk-parallel forward of Falcon-2 (regression, one step
// and decay per value channel) on the tcgen05 tensor cores, bf16 inputs,
// d_k = d_v = 128, chunk 64.
//
// Method: Falcon-2 takes eta and alpha per value channel j, i.e. per row of S
// (page "借鉴40年前的设想！…", 02 (2)); the chunk form is parallel inside a
// chunk and recurrent across chunks (page "Fast Weight Attention：用于持续学
// 习的快速权重注意力", 核心方法 3).  Row j of S runs its own normalised LMS
// recursion s_j <- alpha s_j + eta (y_j - s_j.x) x^T.  Entering a chunk with
// S_0, the errors E[t][j] = y_{t,j} - s_j^{(t-1)}.x_t solve, per channel, the
// unit lower-triangular system
//   E_t + sum_{s<t} e^{G_{t-1}-G_s} eta_s A[t,s] E_s = y_t - e^{G_{t-1}} (S_0 x_t)_j,   A = X X^T,
// with chunk-local G_t = sum_{r<=t} log alpha_r, and then
//   o_t[j]   = e^{G_t} (S_0 q_t)_j + sum_{s<=t} e^{G_t-G_s} eta_s E_s (x_s.q_t)
//   S_end[j] = e^{G_C} S_0[j] + sum_s e^{G_C-G_s} eta_s E_s x_s.
// In the weights of the state update, Z_s = e^{G_C-G_s} eta_s E_s, the
// system reads
//   Z_t = w_t (y_t - e^{G_{t-1}} (S_0 x_t)_j) - (eta_t/alpha_t) sum_{s<t} A[t,s] Z_s,
//   w_t = e^{G_C-G_t} eta_t,
// every coefficient inside the fp32 range, and both remaining sums are
// tensor-core products:
//   o_t[j] = e^{G_t} ((S_0 Q^T)[j][t] + e^{-G_C} (Z^T (P o mask)^T)[j][t]),  P = Q X^T,
//   S_end  = diag(e^{G_C}) S_0 + Z^T X.
// The output form needs G_C > -80 in every channel; a chunk below that
// solves for eta_s E_s with one exponential per term instead.
//
// Rows of S never mix, so a head's channels can be shared out: one block per
// (b, h) walks the chunks for all 128 channels, or, when twice the heads fit
// on the SMs, two blocks per head take 64 channels each (the sample
// normalisation and the key products are then done by both).  S stays in
// fp32 registers (thread: row j, a segment of its columns) with its bf16
// copy in shared memory as the operand of S_0 [X;Q]^T; with 64 channels the
// copy fills both halves of the 128-row operand, so every tensor-memory lane
// quarter holds channel rows.  The per-channel systems are solved by forward
// substitution in blocks of 8 tokens, two threads (lanes of one warp) per
// channel with 128 channels, four with 64: each forms its share of a block's
// sums over the earlier tokens, and all walk it.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc128.cuh"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

__device__ unsigned int g_f2_wait_timeouts;

#ifdef FALCON_TC_DEBUG
// block 0, thread 0: SM cycles per phase summed over the chunks
__device__ long long *g_f2_tim;
#define F2T_INIT()                  \
    long long f2t_acc_[8] = {0};    \
    long long f2t_prev_ = clock64(); \
    const bool f2t_on_ = blockIdx.x == 0 && threadIdx.x == 0
#define F2T(k)                                      \
    do {                                            \
        if (f2t_on_) {                              \
            const long long n_ = clock64();         \
            f2t_acc_[k] += n_ - f2t_prev_;          \
            f2t_prev_ = n_;                         \
        }                                           \
    } while (0)
#define F2T_END()                                                             \
    do {                                                                      \
        if (f2t_on_ && g_f2_tim)                                              \
            for (int i_ = 0; i_ < 8; ++i_) g_f2_tim[i_] = f2t_acc_[i_];        \
    } while (0)
#else
#define F2T_INIT()
#define F2T(k)
#define F2T_END()
#endif

constexpr uint32_t F_IN = 0;          // [X;Q] per K half: half k at 2 TILE k, X rows 0-63, Q rows 64-127
constexpr uint32_t F_V = 4 * TILE;    // values (tile pair)
constexpr uint32_t F_B = 6 * TILE;    // per-channel beta (tile pair)
constexpr uint32_t F_S = 8 * TILE;    // bf16 S_0: K half k at F_S + 2 TILE k (128 rows j)
constexpr uint32_t F_XT = 12 * TILE;  // X^T: 128 rows i x 64 s
constexpr uint32_t F_ZT = 14 * TILE;  // Z^T: 128 rows j x 64 s
constexpr uint32_t F_PM = 16 * TILE;  // P o mask (s <= t): 64 rows t x 64 s
constexpr uint32_t F_G = 17 * TILE;   // fp32 G[t][j] at gidx(t, j)
constexpr int LDA = 68;               // fp32 row stride of A (16-byte rows, conflict-free stores)
constexpr uint32_t F_A = F_G + CH * DD * 4;     // fp32 A[t][s] for s < t, zero above
constexpr uint32_t F_VEC = F_A + CH * LDA * 4;  // |x|^2 [64], 1/(eps+|x|^2) [64], group log sums [256], G_C [128],
                                                // group products [256]
constexpr uint32_t F_BAR = F_VEC + (64 + 64 + 2 * DD + DD + 2 * DD) * 4;
constexpr uint32_t F_SMEM = F_BAR + 64 + 1024;
// tensor memory (512 columns)
constexpr uint32_t C_PA = 0;    // [X;Q] X^T: A rows t (lanes 0-63), P rows t (lanes 64-127); 64 columns
constexpr uint32_t C_S = 64;    // S_0 [X;Q]^T: lanes j; (S_0 X^T)[j][t] in 0-63, (S_0 Q^T)[j][t] in 64-127
constexpr uint32_t C_DS = 192;  // Z^T X: lanes j, columns i
constexpr uint32_t C_I = 320;   // Z^T (P o mask)^T: lanes j, columns t
constexpr float kMinLogDecay = -80.f;

// fp32 G table: row t, column j ^ (t mod 32) (conflict-free along either index)
__device__ __forceinline__ int gidx(int t, int j) { return t * DD + (j ^ (t & 31)); }

// bf16 copy of this thread's state columns seg * SC .. + SC - 1 of row j
// (SC = 64 with 128 channels, 32 with 64 channels, whose rows go to both
// halves of the operand)
template <int NJ>
__device__ __forceinline__ void store_state_image(uint8_t *sm, int j, int seg, const float *S) {
    constexpr int SC = 128 / (256 / NJ);
    const int half = (seg * SC) >> 6, ch0 = ((seg * SC) & 63) >> 3;
#pragma unroll
    for (int c8 = 0; c8 < SC / 8; ++c8) {
        const uint4 u = pack8(&S[c8 * 8]);
        *reinterpret_cast<uint4 *>(sm + F_S + half * 2 * TILE + tc::sw128(j, ch0 + c8)) = u;
        if (NJ == 64) *reinterpret_cast<uint4 *>(sm + F_S + half * 2 * TILE + tc::sw128(j + 64, ch0 + c8)) = u;
    }
}

// a[part * STRIDE] for a compile-time array position a and a runtime part < TPC
template <int TPC, int STRIDE>
__device__ __forceinline__ float pick(const float *a, int part) {
    if constexpr (TPC == 2) {
        return part ? a[STRIDE] : a[0];
    } else {
        return (part & 2) ? ((part & 1) ? a[3 * STRIDE] : a[2 * STRIDE]) : ((part & 1) ? a[STRIDE] : a[0]);
    }
}

// bf16 element (t, s) of the 64-row P o mask tile
__device__ __forceinline__ float pm_get(const uint8_t *sm, int t, int s) {
    return __bfloat162float(
        *reinterpret_cast<const __nv_bfloat16 *>(sm + F_PM + tc::sw128(t, s >> 3) + (uint32_t)(s & 7) * 2));
}

}  // namespace

template <int NJ>
__global__ void __launch_bounds__(NTH, 1) f2_chunk_kernel(FwdParams p, const __grid_constant__ PcMaps maps) {
    constexpr int NSPLIT = DD / NJ;  // blocks per head
    constexpr int NSEG = 256 / NJ;   // threads per channel in the solve and the epilogue
    constexpr int SC = DD / NSEG;    // state columns per thread
    constexpr bool DUP = NJ == 64;   // channel rows in both halves of the 128-row operands
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *Gt = reinterpret_cast<float *>(sm + F_G);
    float *At = reinterpret_cast<float *>(sm + F_A);
    float *sqn = reinterpret_cast<float *>(sm + F_VEC);
    float *rinv = sqn + 64;
    float *hsum = rinv + 64;
    float *gcv = hsum + 2 * DD;
    float *hprod = gcv + DD;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + F_BAR);
    uint64_t *tbar = bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, chalf = warp >> 2, row = quarter * 32 + lane;
    // this thread's tensor-memory lane holds channel jl (of the block's NJ);
    // its segment of that channel's tokens and state columns is seg
    const int jl = row & (NJ - 1), seg = DUP ? 2 * (quarter >> 1) + chalf : chalf;
    const int bh = blockIdx.x / NSPLIT, J0 = (blockIdx.x % NSPLIT) * NJ;
    const int L = p.L, nch = (L + CH - 1) / CH;
    const float lam = p.lambda[bh % p.H];

    // keys (rows c0-1 .. under the prefix pair) and q as [X;Q] per K half, then
    // the block's columns of v and beta (both halves, or the one of its channels)
    auto load_chunk = [&](int c) {
        const int c0 = c * CH, krow = p.pairing == 0 ? c0 - 1 : c0;
        tc::mbar_arrive_expect_tx(tbar, (4 + 2 * (NJ / 64)) * TILE);
        tc::tma_load_3d(sbase + F_IN, &maps.k, 0, krow, bh, tbar);
        tc::tma_load_3d(sbase + F_IN + TILE, &maps.q, 0, c0, bh, tbar);
        tc::tma_load_3d(sbase + F_IN + 2 * TILE, &maps.k, 64, krow, bh, tbar);
        tc::tma_load_3d(sbase + F_IN + 3 * TILE, &maps.q, 64, c0, bh, tbar);
        if constexpr (NJ == DD) {
            load_pair(sbase + F_V, &maps.v, c0, bh, tbar);
            load_pair(sbase + F_B, &maps.beta, c0, bh, tbar);
        } else {
            tc::tma_load_3d(sbase + F_V, &maps.v, J0, c0, bh, tbar);
            tc::tma_load_3d(sbase + F_B, &maps.beta, J0, c0, bh, tbar);
        }
    };
    int issued = 0;  // chunk loads issued (thread 0)
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(tbar, 1);
        tc::fence_mbar_init();
        if (nch > 0) {
            load_chunk(0);
            issued = 1;
        }
    }
    __syncwarp();
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    // S in fp32 registers: thread = (row J0 + jl, columns seg * SC ..)
    float S[SC];
#pragma unroll
    for (int e = 0; e < SC; ++e)
        S[e] = p.init_state ? p.init_state[((size_t)bh * DD + J0 + jl) * DD + seg * SC + e] : 0.f;
    store_state_image<NJ>(sm, jl, seg, S);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);

    bool ok = true;
    uint32_t phase = 0;
    F2T_INIT();
    for (int c = 0; c < nch; ++c) {
        const int c0 = c * CH, nt = min(CH, L - c0);
        ok = tc::mbar_wait_timeout(tbar, (uint32_t)(c & 1), kWaitNs);
        ok = __syncthreads_and(ok);
        if (!ok) break;
        F2T(0);
        // ---- samples, then S_0 [X;Q]^T and [X;Q] X^T on the tensor core
        samples_pair(sm, F_IN, 2 * TILE, p, bh, c == 0, sqn, rinv);
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        F2T(1);
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_gemm(tbase + C_PA, sbase + F_IN, 2 * TILE, sbase + F_IN, 2 * TILE, 2, 64);
            issue_gemm(tbase + C_S, sbase + F_S, 2 * TILE, sbase + F_IN, 2 * TILE, 2, 128);
            tc::mma_commit(bar);
        }
        // ---- decays: thread (token group h, channel jj), TG running log sums and
        //      products in registers; X^T.  F_G then holds e^{G_t} (as products of
        //      the factors), or G_t itself in a chunk whose G_C is -80 or below
        bool unsafe;
        {
            constexpr int NG = 256 / NJ, TG = CH / NG;
            const int h = tid / NJ, jj = tid % NJ;
            float Gl[TG], Pl[TG];
            float acc = 0.f, prod = 1.f;
#pragma unroll
            for (int i = 0; i < TG; ++i) {
                const int t = h * TG + i;
                const float eta = pair_get(sm, F_B, t, jj) * rinv[t];
                const float alpha = fmaxf(1.f - eta * lam, kAlphaFloor);
                acc += __logf(alpha);
                prod *= alpha;
                Gl[i] = acc;
                Pl[i] = prod;
            }
            hsum[h * NJ + jj] = acc;
            hprod[h * NJ + jj] = prod;
            for (int g = warp; g < 32; g += NTH / 32) {
                const int half = g >> 4, rb = (g >> 1) & 7, cb0 = (g & 1) * 4;
                transpose4(sbase + F_IN + half * 2 * TILE, rb, cb0, sbase + F_XT, half * 64);
            }
            __syncthreads();
            float base = 0.f, tot = 0.f, pbase = 1.f;
#pragma unroll
            for (int h2 = 0; h2 < NG; ++h2) {
                const float hs = hsum[h2 * NJ + jj];
                if (h2 < h) {
                    base += hs;
                    pbase *= hprod[h2 * NJ + jj];
                }
                tot += hs;
            }
            unsafe = __syncthreads_or(!(tot > kMinLogDecay)) != 0;
#pragma unroll
            for (int i = 0; i < TG; ++i) Gt[gidx(h * TG + i, jj)] = unsafe ? base + Gl[i] : pbase * Pl[i];
            if (h == 0) gcv[jj] = tot;
        }
        __syncthreads();
        F2T(2);
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        F2T(3);
        tc::fence_after_sync();
        // ---- A (lanes 0-63) -> fp32 rows t, s < t; P (lanes 64-127) -> bf16 P o mask rows t, s <= t
        {
            const int t = row & 63;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16];
                tc::tmem_ld16(tl + C_PA + cs * 16, v);
                tc::tmem_wait_ld();
                if (quarter < 2) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = cs * 16 + i < t ? v[i] : 0.f;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<float4 *>(At + t * LDA + cs * 16 + q4 * 4) =
                            make_float4(v[q4 * 4], v[q4 * 4 + 1], v[q4 * 4 + 2], v[q4 * 4 + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = cs * 16 + i <= t ? v[i] : 0.f;
                    *reinterpret_cast<uint4 *>(sm + F_PM + tc::sw128(t, cs * 2)) = pack8(&v[0]);
                    *reinterpret_cast<uint4 *>(sm + F_PM + tc::sw128(t, cs * 2 + 1)) = pack8(&v[8]);
                }
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        F2T(4);
        tc::fence_after_sync();
        // ---- per-channel systems.  TPC threads per channel, lanes of one warp.
        //      128 channels: warp w takes channels 32 (w & 3) + 16 (w >> 2) .. +15
        //      (inside its tensor-memory lanes), lane l channel ... + l / 2.  64
        //      channels (rows in both lane halves): the four warps of lane
        //      quarters q and q ^ 2 take 8 channels each of 32 (q & 1) .. +31, lane
        //      l channel ... + l / 4.  Each thread of a channel forms 8 / TPC of
        //      the eight sums over the rows before a block of 8 tokens; the
        //      threads swap them and all walk the block.
        if (!unsafe) {
            constexpr int TPC = NSEG, PT = 8 / TPC;
            const int part = lane & (TPC - 1);
            const int slot = DUP ? (warp >> 2) + 2 * (quarter >> 1) : (warp >> 2);
            const int src = (32 / TPC) * slot + lane / TPC;  // the channel's lane inside this quarter
            const int jj = 32 * (DUP ? (quarter & 1) : quarter) + src;
            const float egc = Gt[gidx(CH - 1, jj)];  // e^{G_C}
            float Z[64];
#pragma unroll
            for (int s = 0; s < 64; ++s) Z[s] = 0.f;
#pragma unroll
            for (int tb = 0; tb < 4; ++tb) {
                float xs[16];
                tc::tmem_ld16(tl + C_S + tb * 16, xs);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) xs[i] = __shfl_sync(0xffffffffu, xs[i], src);  // channel jj's row
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int t0 = tb * 16 + hb * 8, tp = t0 + PT * part;  // this thread's PT tokens
                    float r[8], kap[8], cr[8], rm[PT], km[PT];
                    float egp = tp > 0 ? Gt[gidx(tp - 1, jj)] : 1.f;  // e^{G_{t-1}}
#pragma unroll
                    for (int i = 0; i < PT; ++i) {
                        const int t = tp + i;
                        const float eta = pair_get(sm, F_B, t, jj) * rinv[t];
                        const float alpha = fmaxf(1.f - eta * lam, kAlphaFloor);
                        const float eg = Gt[gidx(t, jj)];
                        const float x = pick<TPC, PT>(&xs[hb * 8 + i], part);
                        rm[i] = __fdividef(egc, eg) * eta * (pair_get(sm, F_V, t, jj) - egp * x);
                        km[i] = __fdividef(eta, alpha);
                        egp = eg;
                    }
                    if constexpr (TPC == 2) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float ro = __shfl_xor_sync(0xffffffffu, rm[i], 1);
                            const float ko = __shfl_xor_sync(0xffffffffu, km[i], 1);
                            r[i] = part ? ro : rm[i];
                            r[4 + i] = part ? rm[i] : ro;
                            kap[i] = part ? ko : km[i];
                            kap[4 + i] = part ? km[i] : ko;
                        }
                    } else {
#pragma unroll
                        for (int q2 = 0; q2 < TPC; ++q2)
#pragma unroll
                            for (int i = 0; i < PT; ++i) {
                                r[q2 * PT + i] = __shfl_sync(0xffffffffu, rm[i], (lane & ~(TPC - 1)) | q2);
                                kap[q2 * PT + i] = __shfl_sync(0xffffffffu, km[i], (lane & ~(TPC - 1)) | q2);
                            }
                    }
                    // rows t0 + PT part .. + PT - 1 of this thread, then the others'
                    float cm[PT];
#pragma unroll
                    for (int i = 0; i < PT; ++i) cm[i] = 0.f;
                    const float *arow = At + (t0 + PT * part) * LDA;
#pragma unroll
                    for (int s = 0; s < t0; s += 4) {
#pragma unroll
                        for (int i = 0; i < PT; ++i) {
                            const float4 a = *reinterpret_cast<const float4 *>(arow + i * LDA + s);
                            cm[i] = fmaf(a.x, Z[s], fmaf(a.y, Z[s + 1], fmaf(a.z, Z[s + 2], fmaf(a.w, Z[s + 3], cm[i]))));
                        }
                    }
                    if constexpr (TPC == 2) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float other = __shfl_xor_sync(0xffffffffu, cm[i], 1);
                            cr[i] = part ? other : cm[i];
                            cr[4 + i] = part ? cm[i] : other;
                        }
                    } else {
#pragma unroll
                        for (int q2 = 0; q2 < TPC; ++q2)
#pragma unroll
                            for (int i = 0; i < PT; ++i)
                                cr[q2 * PT + i] = __shfl_sync(0xffffffffu, cm[i], (lane & ~(TPC - 1)) | q2);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float acc = cr[i];
#pragma unroll
                        for (int s = t0; s < t0 + i; ++s) acc = fmaf(At[(t0 + i) * LDA + s], Z[s], acc);
                        Z[t0 + i] = r[i] - kap[i] * acc;
                    }
                }
            }
            // Z^T row jj (and its copy in lanes 64-127 with 64 channels): each
            // thread of the channel 64 / TPC of its columns
            if constexpr (TPC == 2) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint4 lo = pack8(&Z[c4 * 8]), hi = pack8(&Z[32 + c4 * 8]);
                    *reinterpret_cast<uint4 *>(sm + F_ZT + tc::sw128(jj, part * 4 + c4)) = part ? hi : lo;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint4 u0 = pack8(&Z[8 * e]), u1 = pack8(&Z[16 + 8 * e]), u2 = pack8(&Z[32 + 8 * e]),
                                u3 = pack8(&Z[48 + 8 * e]);
                    const uint4 u = (part & 2) ? ((part & 1) ? u3 : u2) : ((part & 1) ? u1 : u0);
                    *reinterpret_cast<uint4 *>(sm + F_ZT + tc::sw128(jj, part * 2 + e)) = u;
                    *reinterpret_cast<uint4 *>(sm + F_ZT + tc::sw128(jj + 64, part * 2 + e)) = u;
                }
            }
        } else if (tid < NJ) {
            // (thread = channel jj = tensor-memory lane)
            const int jj = tid;
            const float gc = gcv[jj];
            float Z[64];
            // F_s = eta_s E_s with one exponential per term (every exponent <= 0),
            // the outputs from it, then Z_s = e^{G_C-G_s} F_s
            float xs[64], F[64];
#pragma unroll
            for (int tb = 0; tb < 4; ++tb) {
                float v[16];
                tc::tmem_ld16(tl + C_S + tb * 16, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) xs[tb * 16 + i] = v[i];
            }
            float Gprev = 0.f;
#pragma unroll 1
            for (int t = 0; t < CH; ++t) {
                const float eta = pair_get(sm, F_B, t, jj) * rinv[t];
                float a = 0.f;
                for (int s = 0; s < t; ++s) a += __expf(Gprev - Gt[gidx(s, jj)]) * At[t * LDA + s] * F[s];
                F[t] = eta * (pair_get(sm, F_V, t, jj) - __expf(Gprev) * xs[t] - a);
                Gprev = Gt[gidx(t, jj)];
            }
#pragma unroll
            for (int tb = 0; tb < 4; ++tb) {
                float v[16];
                tc::tmem_ld16(tl + C_S + 64 + tb * 16, v);  // (S_0 Q^T)[j][t]
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) xs[tb * 16 + i] = v[i];
            }
#pragma unroll 1
            for (int t = 0; t < nt; ++t) {
                const float G = Gt[gidx(t, jj)];
                float o = __expf(G) * xs[t];
                for (int s = 0; s <= t; ++s) o += __expf(G - Gt[gidx(s, jj)]) * pm_get(sm, t, s) * F[s];
                static_cast<__nv_bfloat16 *>(p.out)[((size_t)bh * L + c0 + t) * DD + J0 + jj] = __float2bfloat16_rn(o);
            }
#pragma unroll 1
            for (int s = 0; s < CH; ++s) F[s] *= __expf(gc - Gt[gidx(s, jj)]);
#pragma unroll
            for (int s = 0; s < 64; ++s) Z[s] = F[s];
            // Z^T row jj (and its copy)
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                const uint4 u = pack8(&Z[c8 * 8]);
                *reinterpret_cast<uint4 *>(sm + F_ZT + tc::sw128(jj, c8)) = u;
                if (DUP) *reinterpret_cast<uint4 *>(sm + F_ZT + tc::sw128(jj + 64, c8)) = u;
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        F2T(5);
        // the chunk's inputs are consumed: the next chunk's loads run under the rest
        if (tid == 0 && c + 1 < nch) {
            load_chunk(c + 1);
            ++issued;
        }
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_gemm(tbase + C_DS, sbase + F_ZT, 0, sbase + F_XT, 0, 1, 128);                // Z^T X
            if (!unsafe) issue_gemm(tbase + C_I, sbase + F_ZT, 0, sbase + F_PM, 0, 1, 64);    // Z^T (P o mask)^T
            tc::mma_commit(bar);
        }
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        F2T(6);
        tc::fence_after_sync();
        const float gcj = gcv[jl];
        if (!unsafe) {
            // o_t[J0 + jl] for the segment's tokens t = seg * TPS ..
            constexpr int TPS = CH / NSEG;
            const float ig = __expf(-gcj);
#pragma unroll
            for (int k2 = 0; k2 < TPS / 16; ++k2) {
                const int t0 = seg * TPS + k2 * 16;
                float iv[16], av[16];
                tc::tmem_ld16(tl + C_S + 64 + t0, iv);
                tc::tmem_ld16(tl + C_I + t0, av);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = t0 + i;
                    const float o = Gt[gidx(t, jl)] * fmaf(ig, av[i], iv[i]);
                    if (t < nt)
                        static_cast<__nv_bfloat16 *>(p.out)[((size_t)bh * L + c0 + t) * DD + J0 + jl] =
                            __float2bfloat16_rn(o);
                }
            }
        }
        // S_end = diag(e^{G_C}) S_0 + Z^T X, this thread's columns
        {
            const float g = __expf(gcj);
#pragma unroll
            for (int k4 = 0; k4 < SC / 16; ++k4) {
                float dv[16];
                tc::tmem_ld16(tl + C_DS + seg * SC + k4 * 16, dv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) S[k4 * 16 + i] = fmaf(g, S[k4 * 16 + i], dv[i]);
            }
            store_state_image<NJ>(sm, jl, seg, S);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        F2T(7);
    }
    F2T_END();
    if (ok && p.final_state) {
#pragma unroll
        for (int e = 0; e < SC; ++e) p.final_state[((size_t)bh * DD + J0 + jl) * DD + seg * SC + e] = S[e];
    }
    if (!ok && tid == 0) {
        atomicAdd(&g_f2_wait_timeouts, 1u);
        // a load still in flight must land before the block leaves
        if (issued > 0) (void)tc::mbar_wait_timeout(tbar, (uint32_t)((issued - 1) & 1), kWaitNs);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

int launch_f2_chunk(const FwdParams &p, cudaStream_t s) {
    const bool shape_ok = p.variant == F2 && p.dk == DD && p.dv == DD && p.chunk == CH;
    auto al16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!shape_ok || !al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.beta) || !al16(p.out))
        return 1;
    const int BH = p.B * p.H;
    if (BH <= 0 || p.L <= 0) return 1;
    PcMaps maps;
    if (!make_map(&maps.q, p.q, BH, p.L) || !make_map(&maps.k, p.k, BH, p.L) || !make_map(&maps.v, p.v, BH, p.L) ||
        !make_map(&maps.beta, p.beta, BH, p.L))
        return 1;
    static bool attr_set[64] = {false};
    static int sm_count[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = 148;
    if (dev >= 0 && dev < 64 && attr_set[dev]) {
        sms = sm_count[dev];
    } else {
        cudaFuncSetAttribute(f2_chunk_kernel<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)F_SMEM);
        cudaFuncSetAttribute(f2_chunk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)F_SMEM);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
        if (dev >= 0 && dev < 64) {
            sm_count[dev] = sms;
            attr_set[dev] = true;
        }
    }
    // one block per SM: two blocks per head while they all fit at once
    if (2 * BH <= sms)
        f2_chunk_kernel<64><<<(unsigned)(2 * BH), NTH, F_SMEM, s>>>(p, maps);
    else
        f2_chunk_kernel<DD><<<(unsigned)BH, NTH, F_SMEM, s>>>(p, maps);
    return cudaGetLastError() == cudaSuccess ? 0 : -7;  // FALCON_ERR_LAUNCH
}

#ifdef FALCON_TC_DEBUG
extern "C" int falcon_f2_debug_timer_set(long long *ptr) {
    return cudaMemcpyToSymbol(g_f2_tim, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : -1;
}
#endif

unsigned int f2_wait_timeouts() {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_f2_wait_timeouts, sizeof(v));
    return v;
}

}  // namespace falcon
