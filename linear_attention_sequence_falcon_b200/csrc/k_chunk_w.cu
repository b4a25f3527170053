// k_chunk_w.cu -- chunk-parallel forward of Falcon-3 and Falcon-3A (each
// update uses the B_w most recent samples, one scalar step per token) on the
// tcgen05 tensor cores, bf16 inputs, d_k = d_v = 64, chunk 64, B_w = 2..4.
//
// Method: Falcon-3 takes a mini-batch of the last B_w causal samples per
// update, normalised by their summed energy (page "Fast Weight Attention：用
// 于持续学习的快速权重注意力", 核心方法 2; page "借鉴40年前的设想！…", 02 (2));
// the chunk form is parallel inside chunks and recurrent across them (核心
// 方法 3).  Inside a chunk entered with S_0, sample rows r = 0 .. 63+B_w-1
// hold x_i, y_i for i = c0-B_w+1+r, and token t (0..63) updates with rows
// t .. t+B_w-1 (slot m = r - t):
//   S_t = alpha_t S_{t-1} + eta_t sum_m e_{t,m} x_{t+m}^T,
//   e_{t,m} = y_{t+m} - S_{t-1} x_{t+m}   (Falcon-3A: e_{t,m} = y_{t+m}).
// With chunk-local G_t = sum_{s<=t} log alpha_s, weights z_{t,m} =
// e^{G_C-G_t} eta_t e_{t,m} and their running sums per sample row,
// Zacc_t[r] = sum_{s<t} z_{s,r-s}, the system of C*B_w unknowns is solved in
// token order, per value channel j:
//   z_{t,m} = w_t (y_{t+m} - e^{G_{t-1}} (S_0 x_{t+m})_j) - (eta_t/alpha_t) sum_r' A[t+m][r'] Zacc_t[r'],
//   w_t = e^{G_C-G_t} eta_t,  A = X X^T (rows of the sample Gram),
// and with Zt[r] = sum_t z_{t,r-t} (all of the chunk's tokens):
//   S_end = e^{G_C} S_0 + Zt^T X,
//   o_t   = e^{G_t} ((S_0 Q^T)[j][t] + e^{-G_C} (sum_{r<=t} P[t][r] Zt[r]
//                                             + sum_{k=1}^{B_w-1} P[t][t+k] Zacc_{t+1}[t+k])),
// P = Q X^T.  Every coefficient stays inside the fp32 range while G_C > -80;
// a chunk below that runs its tokens one by one (the recurrence itself).
//
// Both variants form every (head, chunk) unit's effect on the state at once
// and hand it, as a per-chunk image, to the chain kernel of the split
// Falcon-1/1A path, which walks the chunks of each head: w_reg_local_kernel
// (Falcon-3) solves the system for the value channels with S_0 = 0 and for
// the rows of the identity with zero values, giving O0, B, Qt and the
// transition; w_local_kernel (Falcon-3A, no state in its increments) walks
// the value channels alone.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

constexpr int CH = 64;   // chunk
constexpr int DD = 64;   // d_k = d_v
constexpr int NTH = 256;
constexpr int ISSUER = 128;
constexpr int NR = 80;   // sample rows held (64 + B_w - 1 <= 67 used), a multiple of 16
constexpr uint32_t TILE = 8192;  // 64 rows x 128 bytes
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kMinLogDecay = -80.f;

__device__ unsigned int g_w_wait_timeouts;

#ifdef FALCON_TC_DEBUG
// w_reg_local_kernel, block 0, threads 0 and 128: SM cycles per phase summed
// over the block's units
__device__ long long *g_wr_tim;
#define WRT_INIT()                  \
    long long wrt_acc_[8] = {0};    \
    long long wrt_bar_ = 0, wrs_[6] = {0, 0, 0, 0, 0, 0}, wrs0_ = 0; \
    long long wrt_prev_ = clock64(); \
    const bool wrt_on_ = blockIdx.x == 0 && (threadIdx.x == 0 || threadIdx.x == 128)
#define WRT(k)                                      \
    do {                                            \
        if (wrt_on_) {                              \
            const long long n_ = clock64();         \
            wrt_acc_[k] += n_ - wrt_prev_;          \
            wrt_prev_ = n_;                         \
        }                                           \
    } while (0)
#define WRT_END()                                                                              \
    do {                                                                                       \
        if (wrt_on_ && g_wr_tim)                                                               \
            for (int i_ = 0; i_ < 8; ++i_) g_wr_tim[(threadIdx.x ? 8 : 0) + i_] = wrt_acc_[i_]; \
        if (wrt_on_ && g_wr_tim) g_wr_tim[16 + (threadIdx.x ? 1 : 0)] = wrt_bar_;                 \
        if (wrt_on_ && g_wr_tim)                                                               \
            for (int i_ = 0; i_ < 6; ++i_) g_wr_tim[24 + (threadIdx.x ? 6 : 0) + i_] = wrs_[i_];    \
    } while (0)
// cycles a walk thread spends in its per-block barrier
#define WRB(stmt)                                       \
    do {                                                \
        const long long b0_ = wrt_on_ ? clock64() : 0;  \
        stmt;                                           \
        if (wrt_on_) wrt_bar_ += clock64() - b0_;       \
    } while (0)
#define WRS_B()                          \
    do {                                 \
        if (wrt_on_) wrs0_ = clock64();  \
    } while (0)
#define WRS_E(k)                                  \
    do {                                          \
        if (wrt_on_) {                            \
            const long long n_ = clock64();       \
            wrs_[k] += n_ - wrs0_;                \
            wrs0_ = n_;                           \
        }                                         \
    } while (0)
#else
#define WRS_B()
#define WRS_E(k)
#define WRB(stmt) stmt
#define WRT_INIT()
#define WRT(k)
#define WRT_END()
#endif


constexpr int LDA = 68;                 // fp32 Gram rows (samples 0-67)
constexpr int LDZ = 84;                 // fp32 per-row sums: conflict-free float4 along the row
// per-token scalars (floats): sqn[80] beta[64] eta[64] alpha[64] G[64] w[64]
// kappa[64] gm1[64] pband[64*4], then red and misc (each kernel's own size)
constexpr int V_SQN = 0, V_BETA = 80, V_ETA = 144, V_ALPHA = 208, V_G = 272, V_W = 336, V_KAP = 400,
              V_GM1 = 464, V_PB = 528, V_RED = 784, V_MISC = 1296, V_END = 1312;

__device__ __forceinline__ uint4 pack8(const float *f) {
    __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
    __nv_bfloat162 c = __floats2bfloat162_rn(f[4], f[5]);
    __nv_bfloat162 d = __floats2bfloat162_rn(f[6], f[7]);
    uint4 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    u.z = *reinterpret_cast<uint32_t *>(&c);
    u.w = *reinterpret_cast<uint32_t *>(&d);
    return u;
}

__device__ __forceinline__ void unpack8(uint4 u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// byte offset of 8-column group g8 of row r in a 64-row [col/8][row][8] bf16 tile
__device__ __forceinline__ uint32_t rowmajor8(int r, int g8) { return (uint32_t)((g8 * 64 + r) * 16); }

// bf16 element (r, c) of a 128-byte-row swizzled tile
__device__ __forceinline__ float tile_get(const uint8_t *sm, uint32_t off, int r, int c) {
    return __bfloat162float(
        *reinterpret_cast<const __nv_bfloat16 *>(sm + off + tc::sw128(r, c >> 3) + (uint32_t)(c & 7) * 2));
}

// D (+)= A B^T, M = 128, K = 64 (four K=16 slices) from tiles a, b, then
// `extra` more K=16 slices from tiles a1, b1.
__device__ __forceinline__ void issue_k(uint32_t d, uint32_t a, uint32_t b, int N, uint32_t a1 = 0, uint32_t b1 = 0,
                                        int extra = 0) {
    const uint32_t idesc = tc::idesc_bf16(128, N, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
        tc::mma_bf16(d, tc::sdesc_sw128(a + kk * 32, 16, 1024), tc::sdesc_sw128(b + kk * 32, 16, 1024), idesc,
                     kk > 0 ? 1u : 0u);
    for (int kk = 0; kk < extra; ++kk)
        tc::mma_bf16(d, tc::sdesc_sw128(a1 + kk * 32, 16, 1024), tc::sdesc_sw128(b1 + kk * 32, 16, 1024), idesc, 1u);
}

// Transposed copy of four 8x8 blocks: source rows 8*srb.., 16-byte chunks
// cb0..cb0+3 of a 128-byte-row tile -> destination rows 8*(cb0..cb0+3)+i,
// chunk dch.  Whole warp.
__device__ __forceinline__ void transpose_blk(uint32_t src, int srb, int cb0, uint32_t dst, int dch) {
    const int lane = threadIdx.x & 31, m = lane >> 3, i = lane & 7;
    uint32_t r[4];
    tc::ldsm_x4_trans(src + (uint32_t)(srb * 8 + i) * 128u + ((uint32_t)((cb0 + m) ^ i) << 4), r);
    const int drow = (cb0 + m) * 8 + i;
    tc::stsm_x4(dst + (uint32_t)drow * 128u + ((uint32_t)(dch ^ (drow & 7)) << 4), r);
}

struct WMaps {
    CUtensorMap q, k, v;
};

}  // namespace

// ============================================================ Falcon-3A: per-chunk images
namespace {
// shared memory of w_local_kernel (bytes from a 1024-aligned base): only the
// inner-product tiles, so that two blocks share an SM.  The Zt^T operands
// are 128-row A tiles of which rows 64-127 (tensor-memory lanes nobody
// reads) fall on the P o mask tile that follows each.
constexpr uint32_t U_XE = 0;            // sample rows x_r (128 rows); then the image staging
constexpr uint32_t U_VE = 2 * TILE;     // sample rows y_r (128 rows)
constexpr uint32_t U_Q = 4 * TILE;      // q rows t (64 rows; rows 64-127 only read as unused A rows)
constexpr uint32_t U_XT0 = 6 * TILE;    // X^T: rows c, samples 0-63
constexpr uint32_t U_XT1 = 7 * TILE;    // X^T: rows c, samples 64-79
constexpr uint32_t U_ZT0 = 8 * TILE;    // Zt^T: rows j, samples 0-63
constexpr uint32_t U_PM0 = 9 * TILE;    // P o (r <= t): rows t, samples 0-63
constexpr uint32_t U_ZT1 = 10 * TILE;   // Zt^T: rows j, samples 64-79
constexpr uint32_t U_PM1 = 11 * TILE;   // rows t, samples 64-79
constexpr uint32_t U_VEC = 12 * TILE;   // scalars (the V_* layout)
constexpr uint32_t U_BAR = U_VEC + V_END * 4;
constexpr uint32_t U_SMEM = U_BAR + 64 + 1024;
static_assert(2 * (U_SMEM + 1024) <= 228 * 1024, "two blocks per SM");
// tensor memory (256 columns): the band terms; P, whose columns the two
// last products reuse once it has been read out
constexpr uint32_t U_G = 0, U_P = 64, U_DS = 64, U_I = 128;
}  // namespace

// The inner-product family has no state in its increments, so a chunk
// entered with S_0 gives, exactly,
//   O = Qt S_0^T + O0,   S_end = g_C S_0 + B,   Qt = D_g Q,
//   O0[t] = e^{G_t - G_C} (sum_{r<=t} P[t][r] Zt[r] + band_t),   B = Zt^T X,
// and every term but the S_0 ones is formed for all (head, chunk) units at
// once here, one block per unit; the chain kernel of the split Falcon-1A
// path then walks the chunks of a head (the image layout is its own:
// [unused | Qt (K-major, swizzled) | O0^T | B ([col/8][row][8])] and g_C).
// A chunk whose G_C is -80 or below sums O0 with one exponential per term.
template <int BW>
__global__ void __launch_bounds__(NTH, 2)
    w_local_kernel(FwdParams p, const __grid_constant__ WMaps maps, uint8_t *img_ws, float *gc_ws) {
    constexpr int MM = CH + BW - 1;  // sample rows of a chunk
    constexpr uint32_t IMG = 4 * TILE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *vec = reinterpret_cast<float *>(sm + U_VEC);
    float *sqn = vec + V_SQN, *vbeta = vec + V_BETA, *veta = vec + V_ETA, *valpha = vec + V_ALPHA, *vG = vec + V_G,
          *vw = vec + V_W, *pband = vec + V_PB, *misc = vec + V_MISC;
    float *veg = vec + V_KAP;  // e^{G_t} (the slot of the regression family's eta/alpha)
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + U_BAR);
    uint64_t *tbar = bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, chalf = warp >> 2, row = quarter * 32 + lane;
    const int L = p.L, nch = (L + CH - 1) / CH;
    const int u = blockIdx.x, bh = u / nch, c = u - bh * nch, c0 = c * CH, nt = min(CH, L - c0);
    const float lam = p.lambda[bh % p.H];
    const __nv_bfloat16 *betap = static_cast<const __nv_bfloat16 *>(p.beta) + (size_t)bh * L;

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(tbar, 1);
        tc::fence_mbar_init();
        // sample row r holds sample i = c0 - BW + 1 + r: key row i-1 (prefix
        // pair) or i (same-step pair), value row i
        const int r0 = c0 - BW + 1, krow = p.pairing == 0 ? r0 - 1 : r0;
        tc::mbar_arrive_expect_tx(tbar, 5 * TILE);
        tc::tma_load_3d(sbase + U_XE, &maps.k, 0, krow, bh, tbar);
        tc::tma_load_3d(sbase + U_XE + TILE, &maps.k, 0, krow + 64, bh, tbar);
        tc::tma_load_3d(sbase + U_VE, &maps.v, 0, r0, bh, tbar);
        tc::tma_load_3d(sbase + U_VE + TILE, &maps.v, 0, r0 + 64, bh, tbar);
        tc::tma_load_3d(sbase + U_Q, &maps.q, 0, c0, bh, tbar);
    }
    __syncwarp();
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 256);
        tc::tmem_relinquish();
    }
    if (tid < CH) vbeta[tid] = tid < nt ? __bfloat162float(betap[c0 + tid]) : 0.f;
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    bool ok = tc::mbar_wait_timeout(tbar, 0, kWaitNs);
    ok = __syncthreads_and(ok);
    uint32_t phase = 0;
    if (ok) {
        // ---- samples: rows r < MM normalised in place (four threads per row), rows MM..NR-1 zero
        for (int rr = tid >> 2; rr < NR; rr += NTH / 4) {  // a warp's lanes share the trip count
            const int part = tid & 3, i = c0 - BW + 1 + rr;
            float xr[16];
            bool given = false;  // a carried sample, used as given
#pragma unroll
            for (int e = 0; e < 16; ++e) xr[e] = 0.f;
            if (rr < MM) {
                // a continued segment: sample 0 (prefix pair) is the carried phi(k); samples
                // before it come from the carried window, values included
                const bool cx = i == 0 && p.pairing == 0 && p.x_prev != nullptr;
                const float *cw = (i < 0 && i >= -(BW - 1) && p.win)
                                      ? p.win + ((size_t)bh * (BW - 1) + (i + BW - 1)) * (DD + DD)
                                      : nullptr;
                given = cx || cw;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int cc = part * 16 + h2 * 8;
                    if (cx) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) xr[h2 * 8 + e] = p.x_prev[(size_t)bh * DD + cc + e];
                    } else if (cw) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) xr[h2 * 8 + e] = cw[cc + e];
                    } else {
                        unpack8(*reinterpret_cast<const uint4 *>(sm + U_XE + tc::sw128(rr, part * 2 + h2)), &xr[h2 * 8]);
                    }
                }
                if (cw) {
                    float yv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) yv[e] = cw[DD + part * 16 + e];
                    *reinterpret_cast<uint4 *>(sm + U_VE + tc::sw128(rr, part * 2)) = pack8(&yv[0]);
                    *reinterpret_cast<uint4 *>(sm + U_VE + tc::sw128(rr, part * 2 + 1)) = pack8(&yv[8]);
                }
            }
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) ss += xr[e] * xr[e];
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            const float inv = (given || p.phi != 0) ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
#pragma unroll
            for (int e = 0; e < 16; ++e) xr[e] *= inv;
            if (part == 0) sqn[rr] = ss * inv * inv;
            *reinterpret_cast<uint4 *>(sm + U_XE + tc::sw128(rr, part * 2)) = pack8(&xr[0]);
            *reinterpret_cast<uint4 *>(sm + U_XE + tc::sw128(rr, part * 2 + 1)) = pack8(&xr[8]);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        // ---- P = Q X^T over the sample rows
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_k(tbase + U_P, sbase + U_Q, sbase + U_XE, NR);
            tc::mma_commit(bar);
        }
        // ---- per-token steps and decays (warps 0-1), X^T (warps 2-7)
        if (tid < CH) {
            const int t = tid;
            float n = 0.f;
#pragma unroll
            for (int m = 0; m < BW; ++m) n += sqn[t + m];
            float eta, alpha;
            step_and_decay(vbeta[t], n, p.eps, lam, eta, alpha);
            float run = __logf(alpha);  // inclusive sum over the warp
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run += y;
            }
            if (lane == 31) misc[warp] = run;
            veta[t] = eta;
            valpha[t] = alpha;
            vG[t] = run;  // warp-local; warp 1 adds warp 0's total below
        } else {
            for (int g = warp - 2; g < 20; g += 6) {
                const int srb = g >> 1, cb0 = (g & 1) * 4;
                transpose_blk(sbase + U_XE, srb, cb0, srb < 8 ? sbase + U_XT0 : sbase + U_XT1, srb & 7);
            }
        }
        __syncthreads();
        if (tid < CH) {
            const int t = tid;
            const float G = vG[t] + (t >= 32 ? misc[0] : 0.f);
            const float GC = misc[0] + misc[1];
            vw[t] = __expf(GC - G) * veta[t];
            __syncwarp();
            vG[t] = G;
            veg[t] = __expf(G);
            if (t == 0) misc[2] = GC;
        }
        __syncthreads();
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        phase ^= 1;
        ok = __syncthreads_and(ok);
    }
    const float GC = misc[2];
    const bool unsafe = !(GC > kMinLogDecay);
    if (ok) {
        tc::fence_after_sync();
        // ---- P (lanes 0-63) -> P o (r <= t) bf16 and the band P[t][t+k], k = 1 .. BW-1
        if (quarter < 2) {
            const int t = row;
            for (int g = chalf; g < 5; g += 2) {
                float v[16];
                tc::tmem_ld16(tl + U_P + g * 16, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = g * 16 + i, k = r - t;
                    if (k >= 1 && k < BW) pband[t * 4 + k] = v[i];
                    v[i] = r <= t ? v[i] : 0.f;
                }
                const uint32_t dst = g < 4 ? U_PM0 : U_PM1;
                const int ch0 = g < 4 ? g * 2 : 0;
                *reinterpret_cast<uint4 *>(sm + dst + tc::sw128(t, ch0)) = pack8(&v[0]);
                *reinterpret_cast<uint4 *>(sm + dst + tc::sw128(t, ch0 + 1)) = pack8(&v[8]);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        // ---- Zt[r] = sum over the tokens whose window holds row r of w_t y_r, and
        //      the band terms sum_k P[t][t+k] Zacc_{t+1}[t+k] (warps 0-1: thread =
        //      channel j = lane), in blocks of 8 tokens: the sums over rows final
        //      before a block are one batch of dot products, one per row of the
        //      block's windows; only the block's own rows are walked token by token
        if (tid < DD) {
            const int j = tid;
            constexpr int NB = 8, RB = NB + BW - 1;  // tokens and rows of a block
            float zb[RB];                            // rows t0 .. t0+RB-1
#pragma unroll
            for (int k = 0; k < RB; ++k) zb[k] = 0.f;
#pragma unroll 1
            for (int tb = 0; tb < 4; ++tb) {
                float bnd[16];
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int t0 = tb * 16 + hb * NB;
#pragma unroll
                    for (int i = 0; i < NB; ++i) {
                        const int t = t0 + i;
                        const float wt = vw[t];
                        // z_{t,m} lands on row t+m
#pragma unroll
                        for (int m = 0; m < BW; ++m) zb[i + m] += wt * tile_get(sm, U_VE, t + m, j);
                        float bsum = 0.f;
#pragma unroll
                        for (int k = 1; k < BW; ++k) bsum = fmaf(pband[t * 4 + k], zb[i + k], bsum);
                        bnd[hb * NB + i] = bsum;
                    }
                    // rows t0 .. t0+7 are final (bf16 Zt^T row j, 16-byte chunk t0 / 8);
                    // rows t0+8 .. carry into the next block
                    *reinterpret_cast<uint4 *>(sm + U_ZT0 + tc::sw128(j, t0 >> 3)) = pack8(zb);
#pragma unroll
                    for (int k = 0; k < RB; ++k) zb[k] = k + NB < RB ? zb[k + NB] : 0.f;
                }
                tc::tmem_st16(tl + U_G + tb * 16, bnd);
            }
            // rows 64 .. 64+BW-2 end the chunk in registers; samples beyond are zero
            float zt[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) zt[k] = k < BW - 1 ? zb[k] : 0.f;
            *reinterpret_cast<uint4 *>(sm + U_ZT1 + tc::sw128(j, 0)) = pack8(&zt[0]);
            *reinterpret_cast<uint4 *>(sm + U_ZT1 + tc::sw128(j, 1)) = pack8(&zt[8]);
            tc::tmem_wait_st();
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_k(tbase + U_DS, sbase + U_ZT0, sbase + U_XT0, DD, sbase + U_ZT1, sbase + U_XT1, 1);  // Zt^T X
            issue_k(tbase + U_I, sbase + U_ZT0, sbase + U_PM0, CH, sbase + U_ZT1, sbase + U_PM1, 1);   // Zt^T (P o m)^T
            tc::mma_commit(bar);
        }
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        phase ^= 1;
        ok = __syncthreads_and(ok);
    }
    if (ok) {
        tc::fence_after_sync();
        // ---- the image, staged over the consumed sample tiles: Qt at 0, O0^T at
        //      TILE, B at 2 TILE (stage offsets; image offsets one TILE more)
        uint8_t *stg = sm + U_XE;
        // Qt = D_g Q: rows t (t >= nt: zero rows of the tile, kept)
        for (int e = tid; e < CH * 8; e += NTH) {
            const int t = e >> 3, c16 = e & 7;
            float q8[8];
            unpack8(*reinterpret_cast<const uint4 *>(sm + U_Q + tc::sw128(t, c16)), q8);
            const float g = veg[t];
#pragma unroll
            for (int i = 0; i < 8; ++i) q8[i] *= g;
            *reinterpret_cast<uint4 *>(stg + tc::sw128(t, c16)) = pack8(q8);
        }
        if (quarter < 2) {
            const int j = row;
            // O0^T row j, tokens 32 chalf .. + 31
            if (!unsafe) {
                const float ig = __expf(-GC);
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    const int t0 = chalf * 32 + k2 * 16;
                    float iv[16], bv[16], o[16];
                    tc::tmem_ld16(tl + U_I + t0, iv);
                    tc::tmem_ld16(tl + U_G + t0, bv);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = t0 + i < nt ? veg[t0 + i] * (ig * (iv[i] + bv[i])) : 0.f;
                    *reinterpret_cast<uint4 *>(stg + TILE + rowmajor8(j, t0 >> 3)) = pack8(&o[0]);
                    *reinterpret_cast<uint4 *>(stg + TILE + rowmajor8(j, (t0 >> 3) + 1)) = pack8(&o[8]);
                }
            } else {
                // O0[t][j] = sum_{s<=t} e^{G_t-G_s} eta_s sum_m P[t][s+m] y_{s+m}[j], one
                // exponential per term (every exponent <= 0); P from the masked tile
                // (r <= t) and the band (r = t+1 .. t+BW-1)
                for (int g8 = 0; g8 < 4; ++g8) {
                    float o[8];
                    for (int i = 0; i < 8; ++i) {
                        const int t = chalf * 32 + g8 * 8 + i;
                        float acc = 0.f;
                        if (t < nt) {
                            const float Gt = vG[t];
                            for (int s = 0; s <= t; ++s) {
                                float a = 0.f;
#pragma unroll
                                for (int m = 0; m < BW; ++m) {
                                    const int r = s + m;
                                    const float pr = r <= t ? tile_get(sm, r < 64 ? U_PM0 : U_PM1, t, r & 63)
                                                            : pband[t * 4 + (r - t)];
                                    a = fmaf(pr, tile_get(sm, U_VE, r, j), a);
                                }
                                acc = fmaf(__expf(Gt - vG[s]) * veta[s], a, acc);
                            }
                        }
                        o[i] = acc;
                    }
                    *reinterpret_cast<uint4 *>(stg + TILE + rowmajor8(j, chalf * 4 + g8)) = pack8(o);
                }
            }
        }
        // B is staged over the value tile, which the branch above may still read
        __syncthreads();
        if (quarter < 2) {
            const int j = row;
            // B row j = (Zt^T X)[j][.], columns 32 chalf .. + 31
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int i0 = chalf * 32 + k2 * 16;
                float dv[16];
                tc::tmem_ld16(tl + U_DS + i0, dv);
                tc::tmem_wait_ld();
                *reinterpret_cast<uint4 *>(stg + 2 * TILE + rowmajor8(j, i0 >> 3)) = pack8(&dv[0]);
                *reinterpret_cast<uint4 *>(stg + 2 * TILE + rowmajor8(j, (i0 >> 3) + 1)) = pack8(&dv[8]);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            gc_ws[u] = __expf(GC);
            tc::bulk_store(img_ws + (size_t)u * IMG + TILE, sbase + U_XE, 3 * TILE);
            tc::bulk_commit();
            tc::bulk_wait_all();
        }
    } else if (tid == 0) {
        atomicAdd(&g_w_wait_timeouts, 1u);
        (void)tc::mbar_wait_timeout(tbar, 0, kWaitNs);  // the load must land before the block leaves
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}


// ============================================================ Falcon-3: per-chunk images
// The chunk's map S_0 -> (O, S_end) is affine.  Running the chunk's
// computation with S_0 = 0 over the real values gives O0 and B, and with
// S_0 = I and zero values it gives Qt and the transition T:
//   O = Qt S_0^T + O0,   S_end = S_0 T + B.
// w_reg_local_kernel does both at once, one block per (head, chunk), on 128
// rows: rows 0-63 are the value channels (S_0 = 0), rows 64-127 the rows of
// the identity (values zero), so the windowed system is walked for 128
// right-hand sides by warps 0-3 (every tensor-memory lane quarter).  It
// writes the chain kernel's image [(T - g_C I)^T | Qt | O0^T | B] and g_C,
// and the chain of the Falcon-1 path walks the chunks of a head.  A chunk
// whose G_C is -80 or below runs the recurrence token by token on the 128
// rows instead.
namespace {
// two sets of input tiles, so that a block prefetches its next unit while it
// computes this one; each set's x and y rows are then its image staging area
constexpr uint32_t R_XE0 = 0;            // sample rows x_r (128 rows)
constexpr uint32_t R_VE0 = 2 * TILE;     // sample rows y_r (128 rows)
constexpr uint32_t R_Q0 = 4 * TILE;      // q rows t (64 rows; the P product reads the next 64 as unused A rows)
constexpr uint32_t R_XE1 = 5 * TILE, R_VE1 = 7 * TILE, R_Q1 = 9 * TILE;
constexpr uint32_t R_XT0 = 10 * TILE;   // X^T: rows c, samples 0-63
constexpr uint32_t R_XT1 = 11 * TILE;   // X^T: rows c, samples 64-79
constexpr uint32_t R_ZT0 = 12 * TILE;   // Zt^T: 128 rows, samples 0-63
constexpr uint32_t R_ZT1 = 14 * TILE;   // Zt^T: 128 rows, samples 64-79
constexpr uint32_t R_PM0 = 16 * TILE;   // P o (r <= t): rows t, samples 0-63
constexpr uint32_t R_PM1 = 17 * TILE;   // rows t, samples 64-79
constexpr uint32_t R_A = 18 * TILE;                   // fp32 A[r][r'], r < 68
constexpr uint32_t R_ZA = R_A + 68 * LDA * 4;         // fp32 Zacc[row][r], 128 rows (token path: outputs)
constexpr uint32_t R_VEC = R_ZA + 2 * DD * LDZ * 4;   // scalars: the V_* layout up to the band, then
constexpr int RV_RED = V_RED, RV_MISC = V_RED + 2 * 4 * 2 * DD, RV_EG = RV_MISC + 16, RV_END = RV_EG + CH;  // red over 128 rows; e^{G_t}
constexpr uint32_t R_BAR = R_VEC + RV_END * 4;  // MMA barrier, one load barrier per set
constexpr uint32_t R_SMEM = R_BAR + 64 + 1024;
static_assert(R_SMEM <= 227 * 1024, "shared memory");
static_assert(2 * DD * CH <= 2 * DD * LDZ, "token-path outputs fit over Zacc");
// tensor memory (512 columns)
constexpr uint32_t RC_G = 0;     // Gram: lanes r, columns r' (80); then the band terms, lanes row, columns t
constexpr uint32_t RC_P = 96;    // P: lanes t, columns r (80)
constexpr uint32_t RC_DS = 192;  // Zt^T X: lanes row, columns c (64)
constexpr uint32_t RC_I = 256;   // Zt^T (P o mask)^T: lanes row, columns t (64)
}  // namespace

template <int BW>
__global__ void __launch_bounds__(NTH, 1)
    w_reg_local_kernel(FwdParams p, const __grid_constant__ WMaps maps, uint8_t *img_ws, float *gc_ws) {
    constexpr int MM = CH + BW - 1;  // sample rows of a chunk
    constexpr uint32_t IMG = 4 * TILE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *At = reinterpret_cast<float *>(sm + R_A);
    float *Za = reinterpret_cast<float *>(sm + R_ZA);
    float *vec = reinterpret_cast<float *>(sm + R_VEC);
    float *sqn = vec + V_SQN, *vbeta = vec + V_BETA, *veta = vec + V_ETA, *valpha = vec + V_ALPHA, *vG = vec + V_G,
          *vw = vec + V_W, *vkap = vec + V_KAP, *vgm1 = vec + V_GM1, *pband = vec + V_PB, *red = vec + RV_RED,
          *misc = vec + RV_MISC, *veg = vec + RV_EG;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + R_BAR);
    uint64_t *tbar = bar + 1;  // [2] the loads of input set 0 / 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, chalf = warp >> 2, row = quarter * 32 + lane;  // row: 0-127
    const int L = p.L, nch = (L + CH - 1) / CH;
    const int units = p.B * p.H * nch;

    // unit w's inputs into set st: sample row r holds sample i = c0 - BW + 1 + r,
    // key row i-1 (prefix pair) or i (same-step pair), value row i
    auto load_unit = [&](int w, int st) {
        const int wbh = w / nch, wc0 = (w - wbh * nch) * CH;
        const int r0 = wc0 - BW + 1, krow = p.pairing == 0 ? r0 - 1 : r0;
        const uint32_t xe = st ? R_XE1 : R_XE0, ve = st ? R_VE1 : R_VE0, qq = st ? R_Q1 : R_Q0;
        tc::mbar_arrive_expect_tx(&tbar[st], 5 * TILE);
        tc::tma_load_3d(sbase + xe, &maps.k, 0, krow, wbh, &tbar[st]);
        tc::tma_load_3d(sbase + xe + TILE, &maps.k, 0, krow + 64, wbh, &tbar[st]);
        tc::tma_load_3d(sbase + ve, &maps.v, 0, r0, wbh, &tbar[st]);
        tc::tma_load_3d(sbase + ve + TILE, &maps.v, 0, r0 + 64, wbh, &tbar[st]);
        tc::tma_load_3d(sbase + qq, &maps.q, 0, wc0, wbh, &tbar[st]);
    };
    int loads = 0;  // loads issued (thread 0)
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(&tbar[0], 1);
        tc::mbar_init(&tbar[1], 1);
        tc::fence_mbar_init();
        if ((int)blockIdx.x < units) {
            load_unit(blockIdx.x, 0);
            loads = 1;
        }
    }
    __syncwarp();
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    // X^T beyond sample 79 only pads its tile
    for (int e = tid; e < TILE / 16; e += NTH)
        *reinterpret_cast<uint4 *>(sm + R_XT1 + e * 16) = make_uint4(0, 0, 0, 0);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    uint32_t phase = 0;  // MMA-completion parity
    bool ok = true;
    int n = 0;
    // beta of a unit's tokens (threads t < CH), read a unit ahead and widened
    // only when it is stored, so that no thread waits for the load
    auto beta_of = [&](int w) {
        const int wbh = w / nch, wc0 = (w - wbh * nch) * CH;
        return tid < min(CH, L - wc0) ? static_cast<const __nv_bfloat16 *>(p.beta)[(size_t)wbh * L + wc0 + tid]
                                      : __float2bfloat16_rn(0.f);
    };
    __nv_bfloat16 bnext = tid < CH && (int)blockIdx.x < units ? beta_of(blockIdx.x) : __float2bfloat16_rn(0.f);
    WRT_INIT();
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++n) {
    const int set = n & 1;
    const uint32_t R_XE = set ? R_XE1 : R_XE0, R_VE = set ? R_VE1 : R_VE0, R_Q = set ? R_Q1 : R_Q0;
    const int bh = u / nch, c = u - bh * nch, c0 = c * CH, nt = min(CH, L - c0);
    const float lam = p.lambda[bh % p.H];
    if (tid < CH) vbeta[tid] = __bfloat162float(bnext);
    ok = tc::mbar_wait_timeout(&tbar[set], (uint32_t)((n >> 1) & 1), kWaitNs);
    ok = __syncthreads_and(ok);
    WRT(0);
    if (!ok) break;
    if (ok) {
        // ---- samples: rows r < MM normalised in place (four threads per row), rows MM..NR-1 zero
        for (int rr = tid >> 2; rr < NR; rr += NTH / 4) {  // a warp's lanes share the trip count
            const int part = tid & 3, i = c0 - BW + 1 + rr;
            float xr[16];
            bool given = false;  // a carried sample, used as given
#pragma unroll
            for (int e = 0; e < 16; ++e) xr[e] = 0.f;
            if (rr < MM) {
                const bool cx = i == 0 && p.pairing == 0 && p.x_prev != nullptr;
                const float *cw = (i < 0 && i >= -(BW - 1) && p.win)
                                      ? p.win + ((size_t)bh * (BW - 1) + (i + BW - 1)) * (DD + DD)
                                      : nullptr;
                given = cx || cw;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int cc = part * 16 + h2 * 8;
                    if (cx) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) xr[h2 * 8 + e] = p.x_prev[(size_t)bh * DD + cc + e];
                    } else if (cw) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) xr[h2 * 8 + e] = cw[cc + e];
                    } else {
                        unpack8(*reinterpret_cast<const uint4 *>(sm + R_XE + tc::sw128(rr, part * 2 + h2)), &xr[h2 * 8]);
                    }
                }
                if (cw) {
                    float yv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) yv[e] = cw[DD + part * 16 + e];
                    *reinterpret_cast<uint4 *>(sm + R_VE + tc::sw128(rr, part * 2)) = pack8(&yv[0]);
                    *reinterpret_cast<uint4 *>(sm + R_VE + tc::sw128(rr, part * 2 + 1)) = pack8(&yv[8]);
                }
            }
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) ss += xr[e] * xr[e];
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            const float inv = (given || p.phi != 0) ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
#pragma unroll
            for (int e = 0; e < 16; ++e) xr[e] *= inv;
            if (part == 0) sqn[rr] = ss * inv * inv;
            *reinterpret_cast<uint4 *>(sm + R_XE + tc::sw128(rr, part * 2)) = pack8(&xr[0]);
            *reinterpret_cast<uint4 *>(sm + R_XE + tc::sw128(rr, part * 2 + 1)) = pack8(&xr[8]);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        WRT(1);
        // ---- the Gram and P over the sample rows
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_k(tbase + RC_G, sbase + R_XE, sbase + R_XE, NR);
            issue_k(tbase + RC_P, sbase + R_Q, sbase + R_XE, NR);
            tc::mma_commit(bar);
        }
        // ---- per-token steps and decays (warps 0-1), X^T (warps 2-7)
        if (tid < CH) {
            const int t = tid;
            float n = 0.f;
#pragma unroll
            for (int m = 0; m < BW; ++m) n += sqn[t + m];
            float eta, alpha;
            step_and_decay(vbeta[t], n, p.eps, lam, eta, alpha);
            float run = __logf(alpha);  // inclusive sum over the warp
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run += y;
            }
            if (lane == 31) misc[warp] = run;
            veta[t] = eta;
            valpha[t] = alpha;
            vG[t] = run;  // warp-local; warp 1 adds warp 0's total below
        } else {
            for (int g = warp - 2; g < 20; g += 6) {
                const int srb = g >> 1, cb0 = (g & 1) * 4;
                transpose_blk(sbase + R_XE, srb, cb0, srb < 8 ? sbase + R_XT0 : sbase + R_XT1, srb & 7);
            }
        }
        __syncthreads();
        WRT(2);
        if (tid < CH) {
            const int t = tid;
            const float G = vG[t] + (t >= 32 ? misc[0] : 0.f);
            const float GC = misc[0] + misc[1];
            const float Gm = G - __logf(valpha[t]);  // G_{t-1}
            const float eta = veta[t];
            vw[t] = __expf(GC - G) * eta;
            vkap[t] = __fdividef(eta, valpha[t]);
            vgm1[t] = __expf(Gm);
            __syncwarp();
            vG[t] = G;
            veg[t] = __expf(G);
            if (t == 0) misc[2] = GC;
        }
        __syncthreads();
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        WRT(3);
        if (tid == 0 && u + (int)gridDim.x < units) {
            // the other set's last image has been read out by its bulk store
            tc::bulk_wait_read();
            load_unit(u + gridDim.x, set ^ 1);
            ++loads;
        }
        if (tid < CH && u + (int)gridDim.x < units) bnext = beta_of(u + gridDim.x);
    }
    const float GC = misc[2];
    const bool unsafe = !(GC > kMinLogDecay);
    uint8_t *stg = sm + R_XE;  // the image, staged over the consumed sample tiles
    if (ok && !unsafe) {
        tc::fence_after_sync();
        // ---- Gram rows r < 68 (lanes 0-79) -> fp32; P (lanes 0-63) -> P o (r <= t) bf16 and the band
        if (quarter < 3) {
            const int r = row;
            for (int g = chalf; g < 5; g += 2) {
                float v[16];
                tc::tmem_ld16(tl + RC_G + g * 16, v);
                tc::tmem_wait_ld();
                if (r < LDA) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (g * 16 + i < LDA) At[r * LDA + g * 16 + i] = v[i];
                }
            }
        }
        if (quarter < 2) {
            const int t = row;
            for (int g = chalf; g < 5; g += 2) {
                float v[16];
                tc::tmem_ld16(tl + RC_P + g * 16, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = g * 16 + i, k = r - t;
                    if (k >= 1 && k < BW) pband[t * 4 + k] = v[i];
                    v[i] = r <= t ? v[i] : 0.f;
                }
                const uint32_t dst = g < 4 ? R_PM0 : R_PM1;
                const int ch0 = g < 4 ? g * 2 : 0;
                *reinterpret_cast<uint4 *>(sm + dst + tc::sw128(t, ch0)) = pack8(&v[0]);
                *reinterpret_cast<uint4 *>(sm + dst + tc::sw128(t, ch0 + 1)) = pack8(&v[8]);
            }
        }
        if (tid < 2 * DD) {
#pragma unroll
            for (int q4 = 0; q4 < NR / 4; ++q4)
                *reinterpret_cast<float4 *>(Za + tid * LDZ + q4 * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        WRT(4);
        tc::fence_after_sync();
        // ---- the chunk's system in token order for 128 right-hand sides (warps
        //      0-3: thread = row = lane): rows 0-63 the value channels (S_0 = 0),
        //      rows 64-127 the rows of the identity (values zero, (S_0 x_r) = x_r[c]);
        //      in blocks of 8 tokens: the sums over rows final before a block are
        //      one batch of dot products, one per row of the block's windows (every
        //      (token, slot) pair that reads a row starts from its sum); only the
        //      block's own rows, in registers, are walked token by token.  Warps
        //      4-7 form each block's sums over the rows final before the block
        //      ahead of it, while warps 0-3 walk that block; warps 0-3 then add
        //      the rows of the block just walked (the same order of additions)
        constexpr int NB = 8, RB = NB + BW - 1;  // tokens and rows of a block
        static_assert(2 * 2 * RB * 2 * DD * 4 <= 4 * TILE, "the sums fit over the Zt^T tiles");
        float *psum = reinterpret_cast<float *>(sm + R_ZT0);  // [2][2][RB][128] the sums, by block parity and half
        if (tid < 2 * DD) {
            const int rw = tid;
            const bool vrow = rw < DD;  // a value channel; else identity row c = rw - 64
            float *za = Za + rw * LDZ;
            auto yv = [&](int r) { return vrow ? tile_get(sm, R_VE, r, rw) : 0.f; };
            auto sxv = [&](int r) { return vrow ? 0.f : tile_get(sm, R_XE, r, rw - DD); };
            float zb[RB];  // rows t0 .. t0+RB-1
#pragma unroll
            for (int k = 0; k < RB; ++k) zb[k] = 0.f;
            WRS_B();
#pragma unroll 1
            for (int tb = 0; tb < 4; ++tb) {
                float bnd[16];
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    const int t0 = tb * 16 + hb * NB, blk = tb * 2 + hb;
                    // rows r' < t0 are final (in shared memory): the sum over them
                    // of A[t+m][r'] Zacc[r'] depends on t+m only, one sum per row;
                    // rows r' < t0 - NB were summed by warps 4-7 during the last block
                    WRB(tc::named_sync(1, NTH));
                    float crr[RB];
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr)
                        crr[rr] = blk > 0 ? psum[((blk & 1) * 2 * RB + rr) * 2 * DD + rw] +
                                                psum[(((blk & 1) * 2 + 1) * RB + rr) * 2 * DD + rw]
                                          : 0.f;
#pragma unroll
                    for (int q = (t0 >> 2) - NB / 4; q < (t0 >> 2); ++q) {
                        if (q < 0) continue;
                        const float4 z4 = *reinterpret_cast<const float4 *>(za + q * 4);
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) {
                            const float4 a4 = *reinterpret_cast<const float4 *>(At + (t0 + rr) * LDA + q * 4);
                            crr[rr] = fmaf(a4.x, z4.x, fmaf(a4.y, z4.y, fmaf(a4.z, z4.z, fmaf(a4.w, z4.w, crr[rr]))));
                        }
                    }
                    // the block's rows of the right-hand side: y_r on a value row,
                    // (S_0 x_r) = x_r[c] on an identity row
                    float ev[RB];
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) ev[rr] = vrow ? yv(t0 + rr) : sxv(t0 + rr);
                    // crr[R]: the sum for row t0+R over the rows final so far; each
                    // row of the block adds its term once it is final
#pragma unroll
                    for (int i = 0; i < NB; ++i) {
                        const int t = t0 + i;
                        const float wt = vw[t], kt = vkap[t];
                        const float cf = vrow ? wt : -(wt * vgm1[t]);  // w_t, or -w_t e^{G_{t-1}}
                        float cri[BW];
#pragma unroll
                        for (int m = 0; m < BW; ++m) {
                            // rows t0+i .. t+BW-2 still accumulating: registers, their
                            // Gram entries read four at a time
                            const float *arow = At + (t + m) * LDA + t0;
                            float acc = crr[i + m];
#pragma unroll
                            for (int k4 = i / 4; k4 <= (i + BW - 2) / 4; ++k4) {
                                const float4 a4 = *reinterpret_cast<const float4 *>(arow + k4 * 4);
                                const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int k = k4 * 4 + e;
                                    if (k >= i && k <= i + BW - 2) acc = fmaf(av[e], zb[k], acc);
                                }
                            }
                            cri[m] = cf * ev[i + m] - kt * acc;
                        }
                        // z_{t,m} lands on row t+m only after every slot of token t used the old sums
#pragma unroll
                        for (int m = 0; m < BW; ++m) zb[i + m] += cri[m];
                        // row t0+i is final: its term into the sums of the block's later
                        // rows (the Gram is symmetric: row t0+i, columns t0+R)
                        const float *acol = At + t * LDA + t0;
#pragma unroll
                        for (int k4 = (i + 1) / 4; k4 * 4 < RB; ++k4) {
                            const float4 a4 = *reinterpret_cast<const float4 *>(acol + k4 * 4);
                            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int R = k4 * 4 + e;
                                if (R > i && R < RB) crr[R] = fmaf(av[e], zb[i], crr[R]);
                            }
                        }
                        const float4 pb4 = *reinterpret_cast<const float4 *>(pband + t * 4);
                        const float pbv[4] = {pb4.x, pb4.y, pb4.z, pb4.w};
                        float bsum = 0.f;
#pragma unroll
                        for (int k = 1; k < BW; ++k) bsum = fmaf(pbv[k], zb[i + k], bsum);
                        bnd[hb * NB + i] = bsum;
                    }
                    // rows t0 .. t0+7 are final; rows t0+8 .. carry into the next block
#pragma unroll
                    for (int k = 0; k < NB; ++k) za[t0 + k] = zb[k];
#pragma unroll
                    for (int k = 0; k < RB; ++k) zb[k] = k + NB < RB ? zb[k + NB] : 0.f;
                }
                tc::tmem_st16(tl + RC_G + tb * 16, bnd);
            }
            WRS_E(0);
            // rows 64 .. 64+BW-2 end the chunk in registers; samples beyond are zero
#pragma unroll
            for (int k = 0; k < BW - 1; ++k) za[CH + k] = zb[k];
            tc::tmem_wait_st();
            float zr[NR];
#pragma unroll
            for (int q4 = 0; q4 < NR / 4; ++q4) {
                const float4 z4 = *reinterpret_cast<const float4 *>(za + q4 * 4);
                zr[q4 * 4] = z4.x; zr[q4 * 4 + 1] = z4.y; zr[q4 * 4 + 2] = z4.z; zr[q4 * 4 + 3] = z4.w;
            }
            tc::named_sync(2, 2 * DD);  // every row's last sums read before Zt^T covers them
            WRS_E(1);
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8)
                *reinterpret_cast<uint4 *>(sm + R_ZT0 + tc::sw128(rw, c8)) = pack8(&zr[c8 * 8]);
#pragma unroll
            for (int c8 = 0; c8 < 2; ++c8)
                *reinterpret_cast<uint4 *>(sm + R_ZT1 + tc::sw128(rw, c8)) = pack8(&zr[64 + c8 * 8]);
        } else {
            // warps 4-7: at each block's start, the sums for the next block over
            // the rows final now (its t0 - NB rows); a thread takes two rows (rw,
            // rw + 64), warps 4-5 the first half of those rows and warps 6-7 the
            // second, so that each Gram row read serves two right-hand sides
            const int h = tid - 2 * DD, qh = h >> 6, rw = h & (DD - 1);
            const float *za0 = Za + rw * LDZ, *za1 = Za + (rw + DD) * LDZ;
            WRS_B();
#pragma unroll 1
            for (int blk = 0; blk < CH / NB; ++blk) {
                const int t0 = blk * NB;
                WRB(tc::named_sync(1, NTH));
                if (blk + 1 < CH / NB) {
                    float c0r[RB], c1r[RB];
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) c0r[rr] = c1r[rr] = 0.f;
                    const int q0 = qh ? (t0 >> 3) : 0, q1 = qh ? (t0 >> 2) : (t0 >> 3);
#pragma unroll 2
                    for (int q = q0; q < q1; ++q) {
                        const float4 z0 = *reinterpret_cast<const float4 *>(za0 + q * 4);
                        const float4 z1 = *reinterpret_cast<const float4 *>(za1 + q * 4);
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) {
                            const float4 a4 = *reinterpret_cast<const float4 *>(At + (t0 + NB + rr) * LDA + q * 4);
                            c0r[rr] = fmaf(a4.x, z0.x, fmaf(a4.y, z0.y, fmaf(a4.z, z0.z, fmaf(a4.w, z0.w, c0r[rr]))));
                            c1r[rr] = fmaf(a4.x, z1.x, fmaf(a4.y, z1.y, fmaf(a4.z, z1.z, fmaf(a4.w, z1.w, c1r[rr]))));
                        }
                    }
                    float *ps = psum + ((((blk + 1) & 1) * 2 + qh) * RB) * 2 * DD;
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) {
                        ps[rr * 2 * DD + rw] = c0r[rr];
                        ps[rr * 2 * DD + rw + DD] = c1r[rr];
                    }
                }
            }
            WRS_E(0);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        WRT(5);
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_k(tbase + RC_DS, sbase + R_ZT0, sbase + R_XT0, DD, sbase + R_ZT1, sbase + R_XT1, 1);  // Zt^T X
            issue_k(tbase + RC_I, sbase + R_ZT0, sbase + R_PM0, CH, sbase + R_ZT1, sbase + R_PM1, 1);   // Zt^T (P o m)^T
            tc::mma_commit(bar);
        }
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        WRT(6);
        if (ok) {
            tc::fence_after_sync();
            WRS_B();
            // ---- the image, every thread one row (0-127) and half of the tokens
            //      and columns: value rows give O0^T and B, identity rows Qt and
            //      T - g_C I (transposed as they are stored)
            const bool vrow = row < DD;
            const int cc = row - DD;
            const float ig = __expf(-GC);
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int t0 = chalf * 32 + k2 * 16;
                float iv[16], bv[16], o[16];
                tc::tmem_ld16(tl + RC_I + t0, iv);
                tc::tmem_ld16(tl + RC_G + t0, bv);
                tc::tmem_wait_ld();
                WRS_E(5);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = t0 + i;
                    const float sq = vrow ? 0.f : tile_get(sm, R_Q, t, cc);
                    o[i] = t < nt ? veg[t] * fmaf(ig, iv[i] + bv[i], sq) : 0.f;
                }
                if (vrow) {
                    *reinterpret_cast<uint4 *>(stg + 2 * TILE + rowmajor8(row, t0 >> 3)) = pack8(&o[0]);
                    *reinterpret_cast<uint4 *>(stg + 2 * TILE + rowmajor8(row, (t0 >> 3) + 1)) = pack8(&o[8]);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        *reinterpret_cast<__nv_bfloat16 *>(stg + TILE + tc::sw128(t0 + i, cc >> 3) + (uint32_t)(cc & 7) * 2) =
                            __float2bfloat16_rn(o[i]);
                }
                WRS_E(2);
            }
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int i0 = chalf * 32 + k2 * 16;
                float dv[16];
                tc::tmem_ld16(tl + RC_DS + i0, dv);
                tc::tmem_wait_ld();
                if (vrow) {
                    *reinterpret_cast<uint4 *>(stg + 3 * TILE + rowmajor8(row, i0 >> 3)) = pack8(&dv[0]);
                    *reinterpret_cast<uint4 *>(stg + 3 * TILE + rowmajor8(row, (i0 >> 3) + 1)) = pack8(&dv[8]);
                } else {
                    // (T - g_C I)[c][i] = (Zt^T X)[64 + c][i], stored at row i, column c
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        *reinterpret_cast<__nv_bfloat16 *>(stg + tc::sw128(i0 + i, cc >> 3) + (uint32_t)(cc & 7) * 2) =
                            __float2bfloat16_rn(dv[i]);
                }
            }
            WRS_E(3);
        }
    } else if (ok) {
        // ---- a chunk whose decay leaves the fp32 range of the factorised form:
        //      the recurrence token by token on the 128 rows, R_t = alpha_t R_{t-1}
        //      + eta_t sum_m (y_{t+m} - R_{t-1} x_{t+m}) x_{t+m}^T (values zero on
        //      the identity rows), o_t = R_t q_t; thread (row, 32 columns), partial
        //      dot products meeting in `red`, the outputs in fp32 over Zacc
        float *outb = Za;  // [row][t]
        for (int e = tid; e < 2 * DD * CH; e += NTH) outb[e] = 0.f;
        float S[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) S[e] = (row >= DD && chalf * 32 + e == row - DD) ? 1.f : 0.f;
        __syncthreads();
        for (int t = 0; t < nt; ++t) {
            float xm[BW][32];
#pragma unroll
            for (int m = 0; m < BW; ++m) {
                float part = 0.f;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    unpack8(*reinterpret_cast<const uint4 *>(sm + R_XE + tc::sw128(t + m, chalf * 4 + c8)), &xm[m][c8 * 8]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) part = fmaf(S[c8 * 8 + i], xm[m][c8 * 8 + i], part);
                }
                red[(chalf * 4 + m) * 2 * DD + row] = part;
            }
            __syncthreads();
            {
                float e[BW];
#pragma unroll
                for (int m = 0; m < BW; ++m) {
                    const float sxm = red[m * 2 * DD + row] + red[(4 + m) * 2 * DD + row];
                    const float y = row < DD ? tile_get(sm, R_VE, t + m, row) : 0.f;
                    e[m] = y - sxm;
                }
                const float eta = veta[t], alpha = valpha[t];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float u2 = 0.f;
#pragma unroll
                    for (int m = 0; m < BW; ++m) u2 = fmaf(e[m], xm[m][i], u2);
                    S[i] = fmaf(alpha, S[i], eta * u2);
                }
            }
            __syncthreads();
            {
                float part = 0.f;
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    float q8[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + R_Q + tc::sw128(t, chalf * 4 + c8)), q8);
#pragma unroll
                    for (int i = 0; i < 8; ++i) part = fmaf(S[c8 * 8 + i], q8[i], part);
                }
                red[(chalf * 4) * 2 * DD + row] = part;
            }
            __syncthreads();
            if (chalf == 0) outb[row * CH + t] = red[row] + red[4 * 2 * DD + row];
            __syncthreads();
        }
        // the image over the consumed sample tiles
        const bool vrow = row < DD;
        const int cc = row - DD;
        const float g = __expf(GC);
        if (vrow) {
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                // B row j, columns 32 chalf .. ; O0^T row j, tokens 32 chalf ..
                *reinterpret_cast<uint4 *>(stg + 3 * TILE + rowmajor8(row, chalf * 4 + g8)) = pack8(&S[g8 * 8]);
                *reinterpret_cast<uint4 *>(stg + 2 * TILE + rowmajor8(row, chalf * 4 + g8)) =
                    pack8(&outb[row * CH + chalf * 32 + g8 * 8]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int col = chalf * 32 + i;  // (T - g_C I)[c][col] at row col, column c
                *reinterpret_cast<__nv_bfloat16 *>(stg + tc::sw128(col, cc >> 3) + (uint32_t)(cc & 7) * 2) =
                    __float2bfloat16_rn(S[i] - (col == cc ? g : 0.f));
                const int t = chalf * 32 + i;    // Qt[t][c] = (T_t q_t)[c]
                *reinterpret_cast<__nv_bfloat16 *>(stg + TILE + tc::sw128(t, cc >> 3) + (uint32_t)(cc & 7) * 2) =
                    __float2bfloat16_rn(outb[row * CH + t]);
            }
        }
    }
    if (!ok) break;
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    WRS_E(4);
    WRT(7);
    if (tid == 0) {
        gc_ws[u] = __expf(GC);
        tc::bulk_store(img_ws + (size_t)u * IMG, sbase + R_XE, IMG);
        tc::bulk_commit();
    }
    }  // units
    if (tid == 0) {
        tc::bulk_wait_all();
        if (!ok) {
            atomicAdd(&g_w_wait_timeouts, 1u);
            // every load issued must land before the block leaves
            for (int k = max(0, loads - 2); k < loads; ++k)
                (void)tc::mbar_wait_timeout(&tbar[k & 1], (uint32_t)((k >> 1) & 1), kWaitNs);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    WRT_END();
    if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
        cudaGetLastError();
    });
    return fn;
}

// [B*H][L][64] bf16, boxes of 64 rows x 64 columns, 128-byte swizzle, zero fill outside
bool make_map(CUtensorMap *m, const void *base, int BH, int L) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DD, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)DD * 2, (cuuint64_t)L * DD * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int w_sm_count() {
    static int counts[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

// Falcon-3 / Falcon-3A: the per-chunk images, then the chain kernel of the split path
template <int BW>
int launch_wl(const FwdParams &p, const WMaps &maps, cudaStream_t s) {
    const size_t units = (size_t)p.B * p.H * ((p.L + CH - 1) / CH);
    void *ws = nullptr;
    bool owned = false;
    const int wrc = ws_acquire(p.ws_given, p.ws, p.ws_bytes, w_local_ws_bytes(p), s, &ws, &owned);
    if (wrc) return wrc;
    uint8_t *img = static_cast<uint8_t *>(ws);
    float *gc = reinterpret_cast<float *>(img + units * 4 * TILE);
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaFuncSetAttribute(w_local_kernel<BW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)U_SMEM);
        cudaFuncSetAttribute(w_reg_local_kernel<BW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)R_SMEM);
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    if (p.variant == F3)  // persistent: one block per SM
        w_reg_local_kernel<BW><<<(unsigned)std::min<size_t>(units, (size_t)w_sm_count()), NTH, R_SMEM, s>>>(p, maps,
                                                                                                       img, gc);
    else
        w_local_kernel<BW><<<(unsigned)units, NTH, U_SMEM, s>>>(p, maps, img, gc);
    int rc = cudaGetLastError() == cudaSuccess ? 0 : -7;  // FALCON_ERR_LAUNCH
    if (rc == 0) rc = launch_chain_images(p, img, gc, s);
    ws_release(ws, owned, s);
    return rc;
}

}  // namespace

bool w_local_covers(const FwdParams &p) {
    if (!((p.variant == F3 || p.variant == F3A) && p.dk == DD && p.dv == DD && p.chunk == CH && p.window >= 2 && p.window <= 4))
        return false;
    return (size_t)p.B * p.H * ((p.L + CH - 1) / CH) <= 0x7fffffffu;
}

size_t w_local_ws_bytes(const FwdParams &p) {
    const size_t units = (size_t)p.B * p.H * ((p.L + CH - 1) / CH);
    return units * 4 * TILE + units * sizeof(float);
}

int launch_w_chunk(const FwdParams &p, cudaStream_t s) {
    const bool shape_ok = (p.variant == F3 || p.variant == F3A) && p.dk == DD && p.dv == DD && p.chunk == CH &&
                          p.window >= 2 && p.window <= 4;
    auto al16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!shape_ok || !al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.out)) return 1;
    const int BH = p.B * p.H;
    if (BH <= 0 || p.L <= 0) return 1;
    WMaps maps;
    if (!make_map(&maps.q, p.q, BH, p.L) || !make_map(&maps.k, p.k, BH, p.L) || !make_map(&maps.v, p.v, BH, p.L))
        return 1;
    if (!w_local_covers(p)) return 1;
    switch (p.window) {
        case 2: return launch_wl<2>(p, maps, s);
        case 3: return launch_wl<3>(p, maps, s);
        default: return launch_wl<4>(p, maps, s);
    }
}

#ifdef FALCON_TC_DEBUG
extern "C" int falcon_wr_debug_timer_set(long long *ptr) {
    return cudaMemcpyToSymbol(g_wr_tim, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : -1;
}
#endif

unsigned int w_wait_timeouts() {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_w_wait_timeouts, sizeof(v));
    return v;
}

}  // namespace falcon
