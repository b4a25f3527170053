// k_chunk_pc.cu -- chunk-parallel forward of Falcon-2A (inner product, one
// step and decay per value channel) on the tcgen05 tensor cores, bf16
// inputs, d_k = d_v = 128, chunk 64.
//
// Method: Falcon-2A takes eta and alpha per value channel j, i.e. per row of
// S (page "借鉴40年前的设想！…", 02 (2)); the chunk form is parallel inside
// chunks and hands a fixed-size state on (page "Fast Weight Attention：用于持
// 续学习的快速权重注意力", 核心方法 3).  Per channel j, with the chunk-local
// G_{t,j} = sum_{r<=t} log alpha_{r,j}, a chunk entered with S gives
//   o_t[j]  = e^{G_{t,j}} (S q_t)[j] + sum_{s<=t} e^{G_{t,j}-G_{s,j}} eta_{s,j} y_{s,j} (x_s . q_t)
//   S_end   = diag(e^{G_{C,j}}) S + dS,   dS[j][i] = sum_s e^{G_{C,j}-G_{s,j}} eta_{s,j} y_{s,j} x_s[i].
// The inner-product family has no solve, and the state recursion is
// elementwise in j (row j of S only ever scales by its own g_j), so the
// forward is three fully parallel kernels:
//   pc_delta_kernel  one block per (head, chunk): the decays (one thread per
//                    channel and half chunk), W[s][j] = e^{G_C-G_s} eta y,
//                    dS = W^T X as one 128x128x64 product; hands on dS,
//                    g = e^{G_C}, W^T and e^{G_t}
//   pc_scan_kernel   one thread per (head, 16-byte column group): S_c for
//                    every chunk (written as the bf16 operand of the next
//                    kernel), S_{c+1} = g_c S_c + dS_c in fp32, the final state
//   pc_out_kernel    one block per (head, chunk): P = Q X^T and Q S_c^T, then
//                    (P o mask) W, and o = e^{G_t} (Q S_c^T + e^{-G_C} (P o mask) W)
//                    while every channel's G_C stays above -80; below that the
//                    intra-chunk terms are summed one exponential at a time.
// Every tcgen05 operand is K-major with 128-byte rows and the 128-byte
// swizzle; d = 128 rows are two 64-column halves.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc128.cuh"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

constexpr uint32_t DSIMG = DD * DD * 2;        // bf16 dS, row-major [j][i]
__device__ unsigned int g_pc_wait_timeouts;

}  // namespace

// ============================================================ dS kernel
namespace {
constexpr uint32_t D_X = 0;            // raw keys -> X (tile pair) -> W^T (128 rows j x 64 s) once X^T is made;
                                       // with D_V the dS image after the product
constexpr uint32_t D_WT = D_X;
constexpr uint32_t D_V = 2 * TILE;     // values -> W[s][j] = e^{G_C-G_s} eta y in place (tile pair)
constexpr uint32_t D_B = 4 * TILE;     // per-channel beta -> E[s][j] = e^{G_s} in place (tile pair)
constexpr uint32_t D_XT = 6 * TILE;    // X^T: 128 rows i x 64 s
constexpr uint32_t D_VEC = 8 * TILE;   // |x_s|^2 [64], 1/(eps+|x_s|^2) [64], quarter-chunk log-decay sums [4][128]
constexpr uint32_t D_BAR = D_VEC + (64 + 64 + 4 * DD) * 4;
constexpr uint32_t D_SMEM = D_BAR + 64 + 1024;
constexpr uint32_t WTIMG = 2 * TILE;   // W^T image handed to pc_out_kernel
constexpr uint32_t EIMG = 2 * TILE;    // e^{G_t} tile pair handed to pc_out_kernel

// per-unit workspace: S_c image, dS image, W^T image, e^{G_t} pair, g = e^{G_C}
constexpr size_t WS_UNIT = (size_t)SIMG + DSIMG + WTIMG + EIMG + DD * sizeof(float);
struct PcWs {
    uint8_t *simg, *dsimg, *wt, *e;
    float *g;
};
__host__ __device__ inline PcWs pc_ws(void *base, size_t units) {
    uint8_t *b = static_cast<uint8_t *>(base);
    PcWs w;
    w.simg = b;
    w.dsimg = w.simg + units * SIMG;
    w.wt = w.dsimg + units * DSIMG;
    w.e = w.wt + units * WTIMG;
    w.g = reinterpret_cast<float *>(w.e + units * EIMG);
    return w;
}
}  // namespace

// One block per unit (b*H + h, chunk); blockIdx.x = bh * nchunks + c.
// The decays are taken by one thread per (pair of adjacent channels, quarter
// of the chunk), so that every shared-memory access moves a bf16 pair: 16
// log-decays per channel summed in registers, the quarters joined through
// shared memory.  Outputs: dS (bf16 image, the layout of the state operand), g =
// e^{G_C}, and for pc_out_kernel W^T (its intra-chunk operand) and e^{G_t}.
__global__ void __launch_bounds__(NTH, 3) pc_delta_kernel(FwdParams p, const __grid_constant__ PcMaps maps, PcWs ws) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *sqn = reinterpret_cast<float *>(sm + D_VEC);
    float *rinv = sqn + 64;
    float *hsum = rinv + 64;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + D_BAR);
    uint64_t *tbar = bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = p.L, nch = (L + CH - 1) / CH;
    const int u = blockIdx.x, bh = u / nch, c0 = (u - bh * nch) * CH;

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(tbar, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(tbar, 6 * TILE);
        load_pair(sbase + D_X, &maps.k, p.pairing == 0 ? c0 - 1 : c0, bh, tbar);
        load_pair(sbase + D_V, &maps.v, c0, bh, tbar);
        load_pair(sbase + D_B, &maps.beta, c0, bh, tbar);
    }
    __syncwarp();
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 128);
        tc::tmem_relinquish();
    }
    const float lam = p.lambda[bh % p.H];
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    bool ok = tc::mbar_wait_timeout(tbar, 0, kWaitNs);
    ok = __syncthreads_and(ok);
    if (ok) {
        samples_pair(sm, D_X, TILE, p, bh, c0 == 0, sqn, rinv);
        __syncthreads();
        // channels j0, j0+1, tokens 16 hq .. 16 hq + 15: the running sums of log alpha
        const int hq = tid >> 6, j0 = 2 * (tid & 63);
        float Gl0[16], Gl1[16];
        {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int s_ = hq * 16 + i;
                const float2 b2 =
                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + D_B + pair_off(s_, j0)));
                const float ri = rinv[s_];
                a0 += __logf(fmaxf(1.f - b2.x * ri * lam, kAlphaFloor));
                a1 += __logf(fmaxf(1.f - b2.y * ri * lam, kAlphaFloor));
                Gl0[i] = a0;
                Gl1[i] = a1;
            }
            *reinterpret_cast<float2 *>(hsum + hq * DD + j0) = make_float2(a0, a1);
        }
        // X^T, four 8x8 groups per warp
        for (int g = warp; g < 32; g += NTH / 32) {
            const int half = g >> 4, rb = (g >> 1) & 7, cb0 = (g & 1) * 4;
            transpose4(sbase + D_X + half * TILE, rb, cb0, sbase + D_XT, half * 64);
        }
        __syncthreads();
        {
            // G_{s,j} = base_j + Gl (base: the quarters before), G_C = the sum of
            // all four; every exponent below is <= 0
            float base0 = 0.f, base1 = 0.f, tot0 = 0.f, tot1 = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 hs = *reinterpret_cast<const float2 *>(hsum + q * DD + j0);
                if (q < hq) {
                    base0 += hs.x;
                    base1 += hs.y;
                }
                tot0 += hs.x;
                tot1 += hs.y;
            }
            const float tail0 = tot0 - base0, tail1 = tot1 - base1;  // G_C - base
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int s_ = hq * 16 + i;
                const uint32_t off = pair_off(s_, j0);
                __nv_bfloat162 *bp = reinterpret_cast<__nv_bfloat162 *>(sm + D_B + off);
                __nv_bfloat162 *vp = reinterpret_cast<__nv_bfloat162 *>(sm + D_V + off);
                const float2 b2 = __bfloat1622float2(*bp), v2 = __bfloat1622float2(*vp);
                const float ri = rinv[s_];
                *vp = __floats2bfloat162_rn(__expf(tail0 - Gl0[i]) * (b2.x * ri) * v2.x,
                                            __expf(tail1 - Gl1[i]) * (b2.y * ri) * v2.y);
                *bp = __floats2bfloat162_rn(__expf(base0 + Gl0[i]), __expf(base1 + Gl1[i]));
            }
            if (hq == 0)
                *reinterpret_cast<float2 *>(ws.g + (size_t)u * DD + j0) = make_float2(__expf(tot0), __expf(tot1));
        }
        __syncthreads();
        transpose_pair(sbase + D_V, sbase + D_WT);
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        // dS[j][i] = sum_s W^T[j][s] X^T[i][s]
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_gemm(tbase, sbase + D_WT, 0, sbase + D_XT, 0, 1, 128);
            tc::mma_commit(bar);
            tc::bulk_store(ws.wt + (size_t)u * WTIMG, sbase + D_WT, WTIMG);
            tc::bulk_store(ws.e + (size_t)u * EIMG, sbase + D_B, EIMG);
            tc::bulk_commit();
        }
        ok = tc::mbar_wait_timeout(bar, 0, kWaitNs);
        // the W^T image leaves shared memory before dS is staged over it
        if (tid == ISSUER) tc::bulk_wait_read();
        ok = __syncthreads_and(ok);
    }
    if (ok) {
        // dS -> bf16 image over W^T and W (both consumed by the product)
        tc::fence_after_sync();
        const int quarter = warp & 3, chalf = warp >> 2, j = quarter * 32 + lane;
        const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            float v[16];
            tc::tmem_ld16(tl + chalf * 64 + k4 * 16, v);
            tc::tmem_wait_ld();
            *reinterpret_cast<uint4 *>(sm + D_X + chalf * 2 * TILE + tc::sw128(j, k4 * 2)) = pack8(&v[0]);
            *reinterpret_cast<uint4 *>(sm + D_X + chalf * 2 * TILE + tc::sw128(j, k4 * 2 + 1)) = pack8(&v[8]);
        }
        tc::fence_proxy_async();
        __syncthreads();
        if (tid == ISSUER) {
            tc::bulk_store(ws.dsimg + (size_t)u * DSIMG, sbase + D_X, DSIMG);
            tc::bulk_commit();
        }
    } else {
        if (tid == 0) atomicAdd(&g_pc_wait_timeouts, 1u);
        (void)tc::mbar_wait_timeout(tbar, 0, kWaitNs);
    }
    if (tid == ISSUER) tc::bulk_wait_read();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 128);
}

// ============================================================ state scan
// One thread per (b*H + h, 16-byte column group of the state image): the
// state at every chunk start (bf16, in the operand layout of pc_out_kernel:
// two K halves of 128 rows x 128 bytes, swizzled), S_{c+1} = g_c S_c + dS_c
// in fp32 (dS in the same image layout), the final state.  Eight chunks'
// loads are issued ahead of their use.
__global__ void __launch_bounds__(256) pc_scan_kernel(FwdParams p, PcWs ws) {
    const int nch = (p.L + CH - 1) / CH;
    const size_t gidx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t rowid = gidx >> 4;  // bh * 128 + j
    if (rowid >= (size_t)p.B * p.H * DD) return;
    const int i8 = (int)(gidx & 15), j = (int)(rowid % DD);
    const size_t bh = rowid / DD;
    float S[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = p.init_state ? p.init_state[rowid * DD + i8 * 8 + e] : 0.f;
    const uint32_t soff = (uint32_t)(i8 >> 3) * (2 * TILE) + tc::sw128(j, i8 & 7);
    constexpr int AHEAD = 8;
    for (int c = 0; c < nch; c += AHEAD) {
        uint4 d[AHEAD];
        float g[AHEAD];
#pragma unroll
        for (int k = 0; k < AHEAD; ++k) {
            const size_t u = bh * nch + min(c + k, nch - 1);
            d[k] = __ldcs(reinterpret_cast<const uint4 *>(ws.dsimg + u * DSIMG + soff));
            g[k] = ws.g[u * DD + j];
        }
#pragma unroll
        for (int k = 0; k < AHEAD; ++k) {
            if (c + k < nch) {
                const size_t u = bh * nch + c + k;
                *reinterpret_cast<uint4 *>(ws.simg + u * SIMG + soff) = pack8(S);
                float dv[8];
                unpack8(d[k], dv);
#pragma unroll
                for (int e = 0; e < 8; ++e) S[e] = g[k] * S[e] + dv[e];
            }
        }
    }
    if (p.final_state) {
#pragma unroll
        for (int e = 0; e < 8; ++e) p.final_state[rowid * DD + i8 * 8 + e] = S[e];
    }
}

// ============================================================ outputs
namespace {
constexpr uint32_t O_Q0 = 0, O_X0 = TILE, O_Q1 = 2 * TILE, O_X1 = 3 * TILE;  // [Q;X] per K half
constexpr uint32_t O_PM = 0;           // P o mask (rows t) over [Q;X] once the first products are done
constexpr uint32_t O_S = 4 * TILE;     // bf16 S_c: K half k at O_S + 2 TILE k (128 rows j); fallback: fp32 G
constexpr uint32_t O_WT = 8 * TILE;    // W^T image (128 rows j x 64 s); fallback: values (tile pair)
constexpr uint32_t O_E = 10 * TILE;    // e^{G_t} (tile pair); fallback: per-channel beta (tile pair)
constexpr uint32_t O_VEC = 12 * TILE;  // g [128], 1/g [128], |x_s|^2 [64]
constexpr uint32_t O_BAR = O_VEC + (2 * DD + 64) * 4;
constexpr uint32_t O_SMEM = O_BAR + 64 + 1024;
// The factorised form scales the intra-chunk sum by e^{-G_C}: safe while every
// channel keeps G_C > -80, i.e. g = e^{G_C} above e^{-80}.
constexpr float kMinGain = 1.80485139e-35f;

// the fallback's fp32 G table: row s, column j ^ (s mod 32) (conflict-free
// along either index)
__device__ __forceinline__ int gidx(int s, int j) { return s * DD + (j ^ (s & 31)); }
}  // namespace

// One block per unit (b*H + h, chunk).  Tensor memory: [P;A] in columns
// 0-63, then the intra-chunk product in 0-127; Q S_c^T in 128-255.  With
// W[s][j] = e^{G_C-G_s} eta y from pc_delta_kernel,
//   o_t[j] = e^{G_t} ( (Q S_c^T)[t][j] + e^{-G_C} ((P o mask) W)[t][j] ).
// A chunk where some channel decays below e^{-80} reloads values and
// betas and sums the intra-chunk terms one exponential at a time.
__global__ void __launch_bounds__(NTH, 2) pc_out_kernel(FwdParams p, const __grid_constant__ PcMaps maps, PcWs ws) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *gv = reinterpret_cast<float *>(sm + O_VEC);
    float *rg = gv + DD;
    float *sqn = rg + DD;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + O_BAR);
    uint64_t *tbar = bar + 1;
    uint64_t *fbar = bar + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 3);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, chalf = warp >> 2, row = quarter * 32 + lane;
    const int L = p.L, nch = (L + CH - 1) / CH;
    const int u = blockIdx.x, bh = u / nch, c0 = (u - bh * nch) * CH, nt = min(CH, L - c0);

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(tbar, 1);
        tc::mbar_init(fbar, 1);
        tc::fence_mbar_init();
        const int krow = p.pairing == 0 ? c0 - 1 : c0;
        tc::mbar_arrive_expect_tx(tbar, 4 * TILE + SIMG + WTIMG + EIMG + DD * 4);
        tc::tma_load_3d(sbase + O_Q0, &maps.q, 0, c0, bh, tbar);
        tc::tma_load_3d(sbase + O_Q1, &maps.q, 64, c0, bh, tbar);
        tc::tma_load_3d(sbase + O_X0, &maps.k, 0, krow, bh, tbar);
        tc::tma_load_3d(sbase + O_X1, &maps.k, 64, krow, bh, tbar);
        tc::bulk_load(sbase + O_S, ws.simg + (size_t)u * SIMG, SIMG, tbar);
        tc::bulk_load(sbase + O_WT, ws.wt + (size_t)u * WTIMG, WTIMG, tbar);
        tc::bulk_load(sbase + O_E, ws.e + (size_t)u * EIMG, EIMG, tbar);
        tc::bulk_load(sbase + O_VEC, ws.g + (size_t)u * DD, DD * 4, tbar);
    }
    __syncwarp();
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 256);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
    bool ok = tc::mbar_wait_timeout(tbar, 0, kWaitNs);
    ok = __syncthreads_and(ok);
    bool unsafe = false, fb_loading = false;
    if (ok) {
        samples_pair(sm, O_X0, 2 * TILE, p, bh, c0 == 0, sqn);
        bool low = false;
        if (tid < DD) {
            const float g = gv[tid];
            low = !(g > kMinGain);
            rg[tid] = 1.f / g;
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        unsafe = __syncthreads_or(low) != 0;
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_gemm(tbase, sbase + O_Q0, 2 * TILE, sbase + O_X0, 2 * TILE, 2, 64);        // [P ; X X^T]
            issue_gemm(tbase + 128, sbase + O_Q0, 2 * TILE, sbase + O_S, 2 * TILE, 2, 128);  // Q S_c^T
            tc::mma_commit(bar);
        }
        if (unsafe && tid == 0) {
            // values and betas over W^T and e^{G_t}, which this path does not read
            tc::mbar_arrive_expect_tx(fbar, 4 * TILE);
            load_pair(sbase + O_WT, &maps.v, c0, bh, fbar);
            load_pair(sbase + O_E, &maps.beta, c0, bh, fbar);
        }
        fb_loading = unsafe;
        ok = tc::mbar_wait_timeout(bar, 0, kWaitNs);
        ok = __syncthreads_and(ok);
    }
    if (ok && !unsafe) {
        tc::fence_after_sync();
        if (quarter < 2) {  // P o mask (s <= t) -> bf16, rows t
            const int t = row;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16];
                tc::tmem_ld16(tl + cs * 16, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = cs * 16 + i <= t ? v[i] : 0.f;
                *reinterpret_cast<uint4 *>(sm + O_PM + tc::sw128(t, cs * 2)) = pack8(&v[0]);
                *reinterpret_cast<uint4 *>(sm + O_PM + tc::sw128(t, cs * 2 + 1)) = pack8(&v[8]);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_gemm(tbase, sbase + O_PM, 0, sbase + O_WT, 0, 1, 128);  // (P o mask) W
            tc::mma_commit(bar);
        }
        ok = tc::mbar_wait_timeout(bar, 1, kWaitNs);
        ok = __syncthreads_and(ok);
        if (ok && quarter < 2) {
            tc::fence_after_sync();
            const int t = row;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.out) + ((size_t)bh * L + c0 + t) * DD;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int jj = chalf * 64 + k4 * 16;
                float iv[16], av[16], ev[16];
                tc::tmem_ld16(tl + 128 + jj, iv);
                tc::tmem_ld16(tl + jj, av);
                unpack8(*reinterpret_cast<const uint4 *>(sm + O_E + pair_off(t, jj)), &ev[0]);
                unpack8(*reinterpret_cast<const uint4 *>(sm + O_E + pair_off(t, jj + 8)), &ev[8]);
                tc::tmem_wait_ld();
                float o[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] = ev[i] * fmaf(rg[jj + i], av[i], iv[i]);
                if (t < nt) {
                    *reinterpret_cast<uint4 *>(dst + jj) = pack8(&o[0]);
                    *reinterpret_cast<uint4 *>(dst + jj + 8) = pack8(&o[8]);
                }
            }
        }
    } else if (ok) {
        // fallback: o_t[j] = e^{G_t} (Q S_c^T)[t][j] + sum_{s<=t} P[t][s] e^{G_t-G_s} eta_s y_s
        ok = tc::mbar_wait_timeout(fbar, 0, kWaitNs);
        ok = __syncthreads_and(ok);
        fb_loading = !ok;
        if (ok) {
            float *Gt = reinterpret_cast<float *>(sm + O_S);
            const float lam = p.lambda[bh % p.H];
            for (int e = tid; e < CH * DD; e += NTH) {
                const int s_ = e >> 7, j = e & (DD - 1);
                const float n = sqn[s_];
                const float eta = n > 0.f ? __fdividef(pair_get(sm, O_E, s_, j), p.eps + n) : 0.f;
                Gt[gidx(s_, j)] = __logf(fmaxf(1.f - eta * lam, kAlphaFloor));
            }
            __syncthreads();
            if (tid < DD) {
                float G = 0.f;
                for (int s_ = 0; s_ < CH; ++s_) {
                    G += Gt[gidx(s_, tid)];
                    Gt[gidx(s_, tid)] = G;
                }
            }
            __syncthreads();
            tc::fence_after_sync();
            if (quarter < 2) {
                const int t = row;
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.out) + ((size_t)bh * L + c0 + t) * DD;
                float prow[CH];
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    float v[16];
                    tc::tmem_ld16(tl + k4 * 16, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) prow[k4 * 16 + i] = v[i];
                }
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int jj = chalf * 64 + k4 * 16;
                    float iv[16];
                    tc::tmem_ld16(tl + 128 + jj, iv);
                    tc::tmem_wait_ld();
                    float o[16];
                    for (int i = 0; i < 16; ++i) {
                        const int j = jj + i;
                        const float gt = Gt[gidx(t, j)];
                        float intra = 0.f;  // one exponential per term, every exponent <= 0
                        for (int s = 0; s <= t; ++s) {
                            const float n = sqn[s];
                            const float eta = n > 0.f ? __fdividef(pair_get(sm, O_E, s, j), p.eps + n) : 0.f;
                            intra += prow[s] * __expf(gt - Gt[gidx(s, j)]) * eta * pair_get(sm, O_WT, s, j);
                        }
                        o[i] = __expf(gt) * iv[i] + intra;
                    }
                    if (t < nt) {
                        *reinterpret_cast<uint4 *>(dst + jj) = pack8(&o[0]);
                        *reinterpret_cast<uint4 *>(dst + jj + 8) = pack8(&o[8]);
                    }
                }
            }
        }
    }
    if (!ok) {
        if (tid == 0) atomicAdd(&g_pc_wait_timeouts, 1u);
        (void)tc::mbar_wait_timeout(tbar, 0, kWaitNs);
        if (fb_loading) (void)tc::mbar_wait_timeout(fbar, 0, kWaitNs);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
}


bool pc_chunk_covers(const FwdParams &p) {
    if (!(p.variant == F2A && p.dk == DD && p.dv == DD && p.chunk == CH)) return false;
    return (size_t)p.B * p.H * ((p.L + CH - 1) / CH) <= 0x7fffffffu;
}

size_t pc_chunk_ws_bytes(const FwdParams &p) { return (size_t)p.B * p.H * ((p.L + CH - 1) / CH) * WS_UNIT; }

int launch_pc_chunk(const FwdParams &p, cudaStream_t s) {
    auto al16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!pc_chunk_covers(p) || !al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.beta) || !al16(p.out) ||
        (p.final_state && !al16(p.final_state)))
        return 1;
    const int BH = p.B * p.H, nch = (p.L + CH - 1) / CH;
    const size_t units = (size_t)BH * nch;
    PcMaps maps;
    if (!make_map(&maps.q, p.q, BH, p.L) || !make_map(&maps.k, p.k, BH, p.L) || !make_map(&maps.v, p.v, BH, p.L) ||
        !make_map(&maps.beta, p.beta, BH, p.L))
        return 1;
    void *ws = nullptr;
    bool owned = false;
    const int wrc = ws_acquire(p.ws_given, p.ws, p.ws_bytes, pc_chunk_ws_bytes(p), s, &ws, &owned);
    if (wrc) return wrc;
    const PcWs w = pc_ws(ws, units);
    static bool attrs_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs_set[dev]) {
        cudaFuncSetAttribute(pc_delta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)D_SMEM);
        cudaFuncSetAttribute(pc_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)O_SMEM);
        if (dev >= 0 && dev < 64) attrs_set[dev] = true;
    }
    pc_delta_kernel<<<(unsigned)units, NTH, D_SMEM, s>>>(p, maps, w);
    const size_t scan_threads = (size_t)BH * DD * 16;
    pc_scan_kernel<<<(unsigned)((scan_threads + 255) / 256), 256, 0, s>>>(p, w);
    pc_out_kernel<<<(unsigned)units, NTH, O_SMEM, s>>>(p, maps, w);
    const cudaError_t e = cudaGetLastError();
    ws_release(ws, owned, s);
    return e == cudaSuccess ? 0 : -7;  // FALCON_ERR_LAUNCH
}

unsigned int pc_wait_timeouts() {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_pc_wait_timeouts, sizeof(v));
    return v;
}

}  // namespace falcon
