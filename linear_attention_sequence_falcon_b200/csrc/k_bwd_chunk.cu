// k_bwd_chunk.cu -- the backward pass of the chunk-parallel form for Falcon-1
// and Falcon-1A (bf16 inputs, d_k = d_v = 64, chunk 64): gradients of a loss
// with respect to q, k, v, beta and lambda, chunk by chunk in parallel; only
// fixed-size states cross chunk boundaries.
//
// Method: the chunk-parallel form is the one the pages train with ("all
// variants are SSD-compatible and can be trained in the chunk-parallel
// form", page "借鉴40年前的设想！…", 02 (2); chunk-parallel for training,
// page "Fast Weight Attention：用于持续学习的快速权重注意力", 工程落地).
//
// One chunk (tokens t = 0..n-1, chunk-local G_t = sum_{r<=t} log alpha_r,
// g_t = e^{G_t}, G_{-1} = 0, g_C = g_{n-1}) entered with state S0 and left
// with S_end, given dO and G^ = dL/dS_end:
//   forward (regression; inner product: E = Y)
//     A = X X^T, P = Q X^T, M[t,s] = e^{G_{t-1}-G_s} eta_s A[t,s] (s < t)
//     E = (I + M)^{-1} (Y - D_a X S0^T),           D_a = diag(e^{G_{t-1}})
//     O = D_g Q S0^T + (P o Dm) E,                   Dm[t,s] = e^{G_t-G_s} eta_s (s <= t)
//     S_end = g_C S0 + E^T D_w X,                    w_s = e^{G_C-G_s} eta_s
//   backward
//     U  = (P o Dm~)^T dO + D_w~ X G^^T              (Dm, w without eta: Dm~, w~)
//     E^ = T^T D_eta U with T = (I + M)^{-1}, and u = U - M~^T E^
//          (M~ = M without eta; inner product: E^ = eta o U, u = U)
//     dY = E^
//     dQ = D_g dO S0 + K X,                          K = (dO E^T) o Dm
//     dX = K^T Q + D_w E G^ - D_a E^ S0 - (Z + Z^T) X,   Z = (E^ E^T) o Md
//          (inner product: K^T Q + D_w Y G^)
//     u_t = G_t x_t (G_t = dL/dS_t), so per token deta_t = e_t . u_t and
//       dL/dlog alpha_t = F_t - eta_t e_t . u_t, where F_t = <G_t, S_t> obeys
//       F_t = do_t . o_t + F_{t+1} - eta_{t+1} y_{t+1} . u_{t+1} for both
//       families (the transition alpha I - eta x x^T is symmetric); it is
//       summed from the chunk's end, where F = <G^, S_end> + do . o, so no
//       sum runs past a chunk boundary.
//   and through the steps and the samples (per token, in the same kernel):
//     alpha = max(1 - eta lambda, 2^-20) (no gradient on the floor),
//     eta = beta / (eps + |x|^2), x = phi(k) (L2 normalisation or identity).
// T comes from the 16 x 16 diagonal blocks of I + M, inverted by
// substitution (D), and K = D M_o (M_o: M off the diagonal blocks, strictly
// block-lower, so K^4 = 0):  T = (I + K)^{-1} D = (I - K + K^2 - K^3) D.
// The state entering chunk c comes from the forward's chain (S_c), and
//   G^_c = g_C G^_{c+1} - G^_{c+1} Phi'_c^T + dO_c^T Qt_c
// (Phi' and Qt, the forward's per-chunk operators) runs backwards over the
// chunks of a head in bwd_rchain_kernel (four blocks per head, sixteen rows
// of G^ each: the rows do not mix); every chunk's gradients then follow at
// once in bwd_chunk_kernel.  The products are TF32 warp MMAs on fp32
// shared-memory tiles (fp32 accumulation; operands truncated to TF32).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"
#include "warp_tf32.cuh"

namespace falcon {

namespace {

constexpr int CC = 64;        // chunk
constexpr int DD = 64;        // d_k = d_v
constexpr int LD = 72;        // fp32 row stride of the tiles: 8-byte fragment loads are conflict-free
constexpr int TF = CC * LD;   // floats per tile
constexpr uint32_t TILE_B = 8192;           // one bf16 64 x 64 tile of the forward's image
constexpr uint32_t IMG_B = 4 * TILE_B;      // the forward's per-chunk image
constexpr int NTH = 512;       // per-chunk kernel: sixteen warps
constexpr int NWK = NTH / 32;
constexpr int NT = 32 / NWK;          // n-tiles (8 columns) per warp: 16 x 16 output blocks
constexpr int RPWK = CC / NWK;        // token rows per warp in the per-row phases
constexpr int NTILE = 12;     // fp32 tiles of the per-chunk kernel
constexpr int NVEC = 16 * 64; // its per-token vectors
constexpr int RQ = 4;         // reverse-chain blocks per (b, h), 16 rows of G^ each
constexpr int NTHR = 128;
constexpr int LDC = 20;       // row stride of the reverse chain's dO columns
constexpr int NBND = RQ * (NTHR / 32);  // partials of <G^, S_end> per chunk

using wt::each;
using wt::ld16;
using wt::st8;
using wt::tf;
using wt::zero;

// 64 x 64 tile products of this file's row stride and warp count (see warp_tf32.cuh)
template <bool TA, bool TB, bool SK = false>
__device__ __forceinline__ void mma64(const float *A, const float *B, float (&acc)[NT][4], int kb, int ke,
                                      const float *sk = nullptr) {
    wt::mma64<LD, TA, TB, SK, NT>(A, B, acc, kb, ke, sk);
}

// The reverse chain's 16 x 16 block per warp (columns 16 w): acc(r, n) +=
// sum_{k < 64} op(A)(r, k) B[k][n], op(A)(r, k) = TA ? A[k][r] : A[r][k]
// (fp32, row stride lda), B a bf16 64 x 64 tile of the forward's image read
// as it is (128-byte rows, 128-byte swizzle, B[k][n] in row k): ldmatrix.trans
// hands each lane B[k0+2t][n] and B[k0+2t+1][n] packed, exactly the TF32
// fragment in the k-slot order of the A side (slot t <- k0+2t, t+4 <- k0+2t+1),
// for two k-steps and both n-tiles in one instruction.
template <bool TA>
__device__ __forceinline__ void mma16b(const float *A, int lda, uint32_t Bt, float (&acc)[2][4]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
    const int cb = warp * 16;
    const int mi = lane >> 3, ri = lane & 7;  // the 8 x 8 matrix this lane addresses, and its row
#pragma unroll 2
    for (int k0 = 0; k0 < 64; k0 += 16) {
        uint32_t bb[4];  // matrix m: k-half m >> 1, n-tile m & 1
        tc::ldsm_x4_trans(Bt + tc::sw128(k0 + (mi >> 1) * 8 + ri, (cb >> 3) + (mi & 1)), bb);
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
            const int ka = k0 + kh * 8 + 2 * t;
            float a0, a1, a2, a3;
            if (TA) {
                a0 = A[ka * lda + g];
                a1 = A[ka * lda + g + 8];
                a2 = A[(ka + 1) * lda + g];
                a3 = A[(ka + 1) * lda + g + 8];
            } else {
                const float2 u0 = *reinterpret_cast<const float2 *>(A + g * lda + ka);
                const float2 u1 = *reinterpret_cast<const float2 *>(A + (g + 8) * lda + ka);
                a0 = u0.x; a2 = u0.y; a1 = u1.x; a3 = u1.y;
            }
            const uint32_t a[4] = {tf(a0), tf(a1), tf(a2), tf(a3)};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const uint32_t w = bb[kh * 2 + nt];
                const uint32_t b[2] = {w << 16, w & 0xffff0000u};
                tc::mma_tf32(acc[nt], a, b);
            }
        }
    }
}

}  // namespace

// ------------------------------------------------------------ reverse chain
// RQ blocks per (b, h), each owning 16 rows of G^ (row j of G_c depends only
// on row j of G_{c+1} and column j of dO_c).  Walking the chunks from the
// last to the first, at chunk c the block
//   * stores its rows of G^_{c+1} (the gradient of the state the chunk
//     leaves) for the per-chunk kernel, with their inner product with the
//     same rows of S_{c+1} (the state the chunk leaves: the next chunk's
//     entering state, or the forward's final state) as per-warp partials;
//   * forms G^_c = g_C G^_{c+1} + G^_{c+1} (-Phi'_c^T) + dO_c^T Qt_c from the
//     forward's image of the chunk (-Phi'^T and Qt, bf16, swizzled) and g_C,
//     while the next chunk's operands are already on their way (registers).
// Inner-product family: no -Phi'^T term (the image has none).
__global__ void __launch_bounds__(NTHR)
    bwd_rchain_kernel(BwdParams p, const uint8_t *img, const float *gc, const float *states,
                      const float *final_state, float *gend, float *bnd, int nch) {
    extern __shared__ __align__(16) float smr[];
    float *Gh = smr;                 // 16 x LD: this block's rows of G^
    float *dOc = Gh + 16 * LD;       // 64 x LDC: dO of the chunk, this block's 16 columns
    uint8_t *Pb = reinterpret_cast<uint8_t *>(dOc + 64 * LDC);  // bf16 -Phi'^T of the chunk, as in the image
    uint8_t *Qb = Pb + TILE_B;                                   // bf16 Qt of the chunk, as in the image
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool reg = p.variant == F1;
    const size_t bh = blockIdx.x / RQ;
    const int qr = blockIdx.x % RQ, L = p.L;
    const __nv_bfloat16 *dout = static_cast<const __nv_bfloat16 *>(p.dout) + bh * (size_t)L * DD;

    // a chunk's operands in registers; two sets, so that the loads of chunk
    // c - 2 are in flight while chunks c and c - 1 are worked on
    struct Ops {
        uint4 p[4], q[4], d;
        float4 s[2];
        float g;
    };
    auto fetch = [&](int c, Ops &o) {
        const size_t u = bh * nch + c;
        const uint4 *im = reinterpret_cast<const uint4 *>(img + u * IMG_B);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (reg) o.p[j] = im[tid + NTHR * j];
            o.q[j] = im[TILE_B / 16 + tid + NTHR * j];
        }
        const int t = c * CC + (tid >> 1);
        o.d = t < L ? ld16(dout + (size_t)t * DD + 16 * qr + 8 * (tid & 1)) : make_uint4(0u, 0u, 0u, 0u);
        const float *sn = c + 1 < nch ? states + (u + 1) * DD * DD : final_state + bh * DD * DD;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int e = tid + NTHR * j;
            o.s[j] = *reinterpret_cast<const float4 *>(sn + (16 * qr + (e >> 4)) * DD + 4 * (e & 15));
        }
        o.g = gc[u];
    };
    auto step = [&](int c, Ops &o) {
        const size_t u = bh * nch + c;
        __syncthreads();  // the previous products are done with Pb, Qb, dOc; G^ is current
        // the chunk's image tiles to shared memory as they are (16-byte pieces)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int pc = tid + NTHR * j;
            if (reg) *reinterpret_cast<uint4 *>(Pb + pc * 16) = o.p[j];
            *reinterpret_cast<uint4 *>(Qb + pc * 16) = o.q[j];
        }
        st8(dOc + (tid >> 1) * LDC + 8 * (tid & 1), o.d);
        // G^_{c+1} out, and <G^_{c+1}, S_{c+1}> over these rows
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int e = tid + NTHR * j, r = e >> 4, col = 4 * (e & 15);
            const float4 gv = *reinterpret_cast<const float4 *>(Gh + r * LD + col);
            *reinterpret_cast<float4 *>(gend + u * DD * DD + (16 * qr + r) * DD + col) = gv;
            part += gv.x * o.s[j].x + gv.y * o.s[j].y + gv.z * o.s[j].z + gv.w * o.s[j].w;
        }
        part = group_sum<32>(part);
        if (lane == 0) bnd[u * NBND + qr * (NTHR / 32) + warp] = part;
        const float g = o.g;
        if (c >= 2) fetch(c - 2, o);
        __syncthreads();
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (reg) mma16b<false>(Gh, LD, tc::smem_u32(Pb), acc);  // G^ (-Phi'^T)
        mma16b<true>(dOc, LDC, tc::smem_u32(Qb), acc);          // dO^T Qt
        const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = gq + (e >> 1) * 8, col = warp * 16 + nt * 8 + 2 * tq + (e & 1);
                acc[nt][e] += g * Gh[r * LD + col];
            }
        __syncthreads();  // every warp has read G^
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = gq + (e >> 1) * 8, col = warp * 16 + nt * 8 + 2 * tq + (e & 1);
                Gh[r * LD + col] = acc[nt][e];
            }
    };

    // G^ at the end of the sequence: dL/dS_L (or zero)
    for (int e = tid; e < 16 * DD; e += NTHR) {
        const int r = e / DD, i = e % DD;
        Gh[r * LD + i] = p.dstate ? p.dstate[(bh * DD + 16 * qr + r) * DD + i] : 0.f;
    }
    Ops oa, ob;
    fetch(nch - 1, oa);
    if (nch >= 2) fetch(nch - 2, ob);
    for (int c = nch - 1; c >= 0; c -= 2) {
        step(c, oa);
        if (c >= 1) step(c - 1, ob);
    }
}

// ------------------------------------------------------------ per-chunk gradients
// One block per (b, h, chunk).  Makes the chunk's samples, steps and decays
// from k, beta and lambda, then writes dq, dv, dk, dbeta of its tokens (dk of
// the key rows its samples came from) and adds its share of dlambda.
__global__ void __launch_bounds__(NTH, 1)
    bwd_chunk_kernel(BwdParams p, const float *states, const float *gend, const float *bnd, int nch) {
    extern __shared__ __align__(16) float sm[];
    float *X = sm, *Q = X + TF, *Y = Q + TF, *dO = Y + TF, *S0 = dO + TF, *Gh = S0 + TF;
    float *MT = Gh + TF;  // e^{G_{t-1}-G_s} A[t,s] (s < t); later Z
    float *PD = MT + TF;  // e^{G_t-G_s} P[t,s] (s <= t); later K
    float *E = PD + TF;   // K (inverse); the residuals R, then E
    float *U = E + TF;    // K^2 (inverse); U, then u; then dX
    float *Eh = U + TF;   // D (inverse); eta o U, then E^
    float *T = Eh + TF;   // (I + M)^{-1}
    float *vec = T + TF;
    float *vG = vec, *veta = vG + 64, *valpha = veta + 64, *vn = valpha + 64, *vinv = vn + 64, *vbeta = vinv + 64;
    float *vred = vbeta + 64;  // [NWK / 4][64] row partials of do . o
    float *va = vred + 4 * 64, *vx = va + 64, *vdga = vx + 64, *vdeta = vdga + 64, *vw = vdeta + 64;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool reg = p.variant == F1;
    const int L = p.L;
    const size_t bh = blockIdx.x / nch;
    const int c = blockIdx.x % nch, t0 = c * CC, n = min(CC, L - t0);
    const float lam = p.lambda[bh % p.H];
    const size_t row0 = bh * (size_t)L + t0;  // first token of the chunk in [B*H*L]
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(p.q) + row0 * DD;
    const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v) + row0 * DD;
    const __nv_bfloat16 *dout = static_cast<const __nv_bfloat16 *>(p.dout) + row0 * DD;
    const __nv_bfloat16 *kh = static_cast<const __nv_bfloat16 *>(p.k) + bh * (size_t)L * DD;
    const __nv_bfloat16 *bt = static_cast<const __nv_bfloat16 *>(p.beta) + row0;
    const size_t u = bh * nch + c;
    const float4 *s0 = reinterpret_cast<const float4 *>(states + u * DD * DD);
    const float4 *ge = reinterpret_cast<const float4 *>(gend + u * DD * DD);

    // ---- inputs: every load in flight first (rows past the sequence end are zero)
    constexpr int NP = 512 / NTH, NF = 1024 / NTH;  // bf16 pieces and fp32 float4 per thread and tile
    uint4 lq[NP], lv[NP], ldo[NP];
    float4 ls[NF], lg[NF];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int e = tid + NTH * j;  // 16-byte piece: row e / 8, columns 8 (e % 8)..
        const bool in = (e >> 3) < n;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        lq[j] = in ? ld16(q + 8 * e) : z;
        lv[j] = in ? ld16(v + 8 * e) : z;
        ldo[j] = in ? ld16(dout + 8 * e) : z;
    }
#pragma unroll
    for (int j = 0; j < NF; ++j) {
        ls[j] = s0[tid + NTH * j];
        lg[j] = ge[tid + NTH * j];
    }
    // samples x_t = phi(k_{t-1}) (prefix pair; phi(k_t) same-step): one warp per row
    uint32_t kw[RPWK];
    float bv[RPWK];
#pragma unroll
    for (int i = 0; i < RPWK; ++i) {
        const int r = warp * RPWK + i, t = t0 + r, kr = p.pairing == 0 ? t - 1 : t;
        kw[i] = (r < n && kr >= 0) ? *reinterpret_cast<const uint32_t *>(kh + (size_t)kr * DD + 2 * lane) : 0u;
        bv[i] = r < n ? __bfloat162float(bt[r]) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < RPWK; ++i) {
        const int r = warp * RPWK + i;
        const float x0 = __uint_as_float(kw[i] << 16), x1 = __uint_as_float(kw[i] & 0xffff0000u);
        const float ss = group_sum<32>(x0 * x0 + x1 * x1);
        const float inv = p.phi != 0 ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
        *reinterpret_cast<float2 *>(X + r * LD + 2 * lane) = make_float2(x0 * inv, x1 * inv);
        if (lane == 0) {
            const float nn = ss * inv * inv;  // the sample's energy (0: no sample)
            float eta = 0.f, alpha = 1.f;
            if (r < n) step_and_decay(bv[i], nn, p.eps, lam, eta, alpha);
            veta[r] = eta;
            valpha[r] = alpha;
            vn[r] = nn;
            vinv[r] = inv;
            vbeta[r] = bv[i];
        }
    }
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int e = tid + NTH * j, off = (e >> 3) * LD + 8 * (e & 7);
        st8(Q + off, lq[j]);
        st8(Y + off, lv[j]);
        st8(dO + off, ldo[j]);
    }
#pragma unroll
    for (int j = 0; j < NF; ++j) {
        const int e = tid + NTH * j, off = (e >> 4) * LD + 4 * (e & 15);
        *reinterpret_cast<float4 *>(S0 + off) = ls[j];
        *reinterpret_cast<float4 *>(Gh + off) = lg[j];
    }
    __syncthreads();
    // chunk-local cumulative log decay (one warp)
    if (warp == 0) {
        float la[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) la[h2] = __logf(valpha[lane + 32 * h2]);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const float y = __shfl_up_sync(0xffffffffu, la[h2], o);
                if (lane >= o) la[h2] += y;
            }
        }
        la[1] += __shfl_sync(0xffffffffu, la[0], 31);
        vG[lane] = la[0];
        vG[lane + 32] = la[1];
    }
    __syncthreads();
    const float GC = vG[CC - 1];
    auto Gm1 = [&](int t) { return t > 0 ? vG[t - 1] : 0.f; };
    const int rb = (warp & 3) * 16, cb = (warp >> 2) * 8 * NT;
    const bool above = cb > rb + 15;  // this warp's output block lies above the diagonal

    float acc[NT][4], acc2[NT][4];
    // ---- A and P, masked with their decays (no steps)
    zero(acc);
    if (!above) mma64<false, true>(X, X, acc, 0, 64);
    each(acc, [&](int r, int s, float &val) { MT[r * LD + s] = s < r ? __expf(Gm1(r) - vG[s]) * val : 0.f; });
    zero(acc);
    if (!above) mma64<false, true>(Q, X, acc, 0, 64);
    each(acc, [&](int r, int s, float &val) { PD[r * LD + s] = s <= r ? __expf(vG[r] - vG[s]) * val : 0.f; });
    __syncthreads();

    if (reg) {
        // ---- T = (I + M)^{-1}.  D: the diagonal blocks' inverses, one column
        //      of a block per thread (threads 0-63); the rest of D is zero
        if (tid < 64) {
            const int o = (tid >> 4) * 16, j = tid & 15;
            float col[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float s = i == j ? 1.f : 0.f;
#pragma unroll
                for (int s2 = 0; s2 < i; ++s2) s -= MT[(o + i) * LD + o + s2] * veta[o + s2] * col[s2];
                col[i] = s;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) Eh[(o + i) * LD + o + j] = col[i];
        } else {
            for (int e = tid - 64; e < CC * CC; e += NTH - 64) {
                const int r = e >> 6, s = e & 63;
                if ((r >> 4) != (s >> 4)) Eh[r * LD + s] = 0.f;
            }
        }
        __syncthreads();
        // K = D M_o: (D M~)[r][s] eta_s on the blocks below the diagonal (D reads its own block only)
        zero(acc);
        mma64<false, false>(Eh, MT, acc, rb, rb + 16);
        each(acc, [&](int r, int s, float &val) { E[r * LD + s] = (s >> 4) < (r >> 4) ? val * veta[s] : 0.f; });
        __syncthreads();
        // K^2 (K[r][k] = 0 for k >= the row's block start)
        zero(acc);
        if (rb > 0) mma64<false, false>(E, E, acc, 0, rb);
        each(acc, [&](int r, int s, float &val) { U[r * LD + s] = val; });
        __syncthreads();
        // I - K + K^2 - K^3
        zero(acc);
        if (rb > 0) mma64<false, false>(E, U, acc, 0, rb);
        each(acc, [&](int r, int s, float &val) {
            T[r * LD + s] = (r == s ? 1.f : 0.f) - E[r * LD + s] + U[r * LD + s] - val;
        });
        __syncthreads();  // K and K^2 are read; the sum is whole
        // T = (I - K + K^2 - K^3) D: each warp reads only the block of the sum it writes
        zero(acc);
        {
            const int ke = min(cb + 8 * NT, rb + 16);
            if (ke > cb) mma64<false, false>(T, Eh, acc, cb, ke);
        }
        __syncwarp();
        each(acc, [&](int r, int s, float &val) { T[r * LD + s] = val; });
    }
    // ---- U = w~ (X G^^T); regression: R = Y - D_a X S0^T
    zero(acc);
    mma64<false, true>(X, Gh, acc, 0, 64);
    each(acc, [&](int r, int j, float &val) { U[r * LD + j] = __expf(GC - vG[r]) * val; });
    if (reg) {
        zero(acc);
        mma64<false, true>(X, S0, acc, 0, 64);
        each(acc, [&](int r, int j, float &val) { E[r * LD + j] = Y[r * LD + j] - __expf(Gm1(r)) * val; });
    }
    __syncthreads();
    // ---- U += (P o Dm~)^T dO (P o Dm~ lower: k >= r); regression: E = T R (T lower: k <= r)
    zero(acc);
    mma64<true, false>(PD, dO, acc, rb, 64);
    if (reg) {
        zero(acc2);
        mma64<false, false>(T, E, acc2, 0, rb + 16);
    }
    __syncthreads();  // every warp has read R
    each(acc, [&](int r, int j, float &val) {
        const float uu = U[r * LD + j] + val;
        U[r * LD + j] = uu;
        Eh[r * LD + j] = veta[r] * uu;
    });
    if (reg) each(acc2, [&](int r, int j, float &val) { E[r * LD + j] = val; });
    __syncthreads();
    if (reg) {
        // E^ = T^T (eta o U) (T^T upper: k >= r); then u = U - M~^T E^
        zero(acc);
        mma64<true, false>(T, Eh, acc, rb, 64);
        __syncthreads();
        each(acc, [&](int r, int j, float &val) { Eh[r * LD + j] = val; });
        __syncthreads();
        zero(acc);
        mma64<true, false>(MT, Eh, acc, rb, 64);
        each(acc, [&](int r, int j, float &val) { U[r * LD + j] -= val; });
        __syncthreads();
    }
    const float *Ef = reg ? E : Y;  // the residuals (inner product: the targets)
    // ---- O = D_g Q S0^T + (P o Dm~) D_eta E: do . o per token (row partials of the two column halves)
    zero(acc);
    mma64<false, true>(Q, S0, acc, 0, 64);
    each(acc, [&](int r, int j, float &val) { val *= __expf(vG[r]); });
    mma64<false, false, true>(PD, Ef, acc, 0, rb + 16, veta);
    {
        float part[2] = {0.f, 0.f};  // rows rb + g and rb + g + 8
        each(acc, [&](int r, int j, float &val) { part[((r & 15) >> 3)] += dO[r * LD + j] * val; });
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            part[h2] += __shfl_xor_sync(0xffffffffu, part[h2], 1);
            part[h2] += __shfl_xor_sync(0xffffffffu, part[h2], 2);
        }
        if ((lane & 3) == 0) {
            const int g = lane >> 2;
            vred[(warp >> 2) * 64 + rb + g] = part[0];
            vred[(warp >> 2) * 64 + rb + g + 8] = part[1];
        }
    }
    // ---- K = (dO E^T) o Dm, over P o Dm once every warp has formed its O
    zero(acc2);
    if (!above) mma64<false, true>(dO, Ef, acc2, 0, 64);
    __syncthreads();
    each(acc2, [&](int r, int s, float &val) {
        PD[r * LD + s] = s <= r ? __expf(vG[r] - vG[s]) * veta[s] * val : 0.f;
    });
    // ---- per-token terms, one warp per row: deta = e . u, and the pieces of
    //      dL/dlog alpha (do . o - eta y . u summed from the chunk's end; eta (y - e) . u)
#pragma unroll 2
    for (int i = 0; i < RPWK; ++i) {
        const int r = warp * RPWK + i;
        const float2 uu = *reinterpret_cast<const float2 *>(U + r * LD + 2 * lane);
        const float2 yy = *reinterpret_cast<const float2 *>(Y + r * LD + 2 * lane);
        const float2 ee = *reinterpret_cast<const float2 *>(Ef + r * LD + 2 * lane);
        const float yu = group_sum<32>(yy.x * uu.x + yy.y * uu.y);
        const float eu = group_sum<32>(ee.x * uu.x + ee.y * uu.y);
        if (lane == 0) {
            const bool in = r < n;
            float a = 0.f;
#pragma unroll
            for (int q4 = 0; q4 < NWK / 4; ++q4) a += vred[64 * q4 + r];
            va[r] = in ? a - veta[r] * yu : 0.f;
            vx[r] = in ? veta[r] * (yu - eu) : 0.f;
            vdeta[r] = eu;
        }
    }
    // dv = E^
    for (int e = tid; e < n * (DD / 2); e += NTH) {
        const int r = e / (DD / 2), j = 2 * (e % (DD / 2));
        *reinterpret_cast<float2 *>(p.dv_out + (row0 + r) * DD + j) =
            *reinterpret_cast<const float2 *>(Eh + r * LD + j);
    }
    // ---- Z = (E^ E^T) o Md over the consumed M (regression)
    if (reg) {
        zero(acc2);
        if (!above) mma64<false, true>(Eh, E, acc2, 0, 64);
    }
    __syncthreads();  // K is complete; M is free; the per-token terms are in place
    if (warp == 0) {
        // the suffix sum over the chunk of do . o - eta y . u, plus <G^, S_end>
        float bnd_ = lane < NBND ? bnd[u * NBND + lane] : 0.f;
        bnd_ = group_sum<32>(bnd_);
        float s1 = va[63 - lane], s0_ = va[31 - lane];  // rows 63 - lane and 31 - lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y1 = __shfl_up_sync(0xffffffffu, s1, o), y0 = __shfl_up_sync(0xffffffffu, s0_, o);
            if (lane >= o) {
                s1 += y1;
                s0_ += y0;
            }
        }
        s0_ += __shfl_sync(0xffffffffu, s1, 31);  // rows 0-31 also take every row of 32-63
        vdga[63 - lane] = s1 + bnd_ + vx[63 - lane];
        vdga[31 - lane] = s0_ + bnd_ + vx[31 - lane];
    }
    if (reg)
        each(acc2, [&](int r, int s, float &val) {
            MT[r * LD + s] = s < r ? __expf(Gm1(r) - vG[s]) * veta[s] * val : 0.f;
        });
    // ---- dQ = D_g dO S0 + K X (K lower: k <= r)
    zero(acc);
    mma64<false, false>(dO, S0, acc, 0, 64);
    each(acc, [&](int r, int i, float &val) { val *= __expf(vG[r]); });
    mma64<false, false>(PD, X, acc, 0, rb + 16);
    {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int r = rb + g + 8 * h2;
                if (r < n)
                    *reinterpret_cast<float2 *>(p.dq + (row0 + r) * DD + cb + nt * 8 + 2 * t) =
                        make_float2(acc[nt][2 * h2], acc[nt][2 * h2 + 1]);
            }
    }
    __syncthreads();  // Z written
    // ---- dX = K^T Q + D_w E G^ - D_a E^ S0 - (Z + Z^T) X
    zero(acc);
    mma64<true, false>(PD, Q, acc, rb, 64);
    zero(acc2);
    mma64<false, false>(Ef, Gh, acc2, 0, 64);
    each(acc2, [&](int r, int i, float &val) { val *= __expf(GC - vG[r]) * veta[r]; });
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] += acc2[nt][e];
    if (reg) {
        zero(acc2);
        mma64<false, false>(Eh, S0, acc2, 0, 64);
        each(acc2, [&](int r, int i, float &val) { val *= __expf(Gm1(r)); });
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] -= acc2[nt][e];
        zero(acc2);
        mma64<false, false>(MT, X, acc2, 0, rb + 16);  // Z X (Z strictly lower)
        mma64<true, false>(MT, X, acc2, rb, 64);       // Z^T X
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] -= acc2[nt][e];
    }
    each(acc, [&](int r, int i, float &val) { U[r * LD + i] = val; });  // dX over u (consumed)
    __syncthreads();
    // ---- per token, one warp per row: dlog alpha -> dalpha -> deta -> dbeta and the
    //      energy's share; then dk of the key row the sample came from (normaliser, phi)
    float dl = 0.f;  // this warp's share of dL/dlambda
    for (int i = 0; i < RPWK; ++i) {
        const int r = warp * RPWK + i;
        if (r >= n) break;
        const int t = t0 + r, kr = p.pairing == 0 ? t - 1 : t;
        const float a = valpha[r], et = veta[r], nn = vn[r];
        const float dalpha = vdga[r] / a;
        float d = vdeta[r];
        if (1.f - et * lam > kAlphaFloor) {
            d -= lam * dalpha;
            dl -= et * dalpha;
        }
        if (lane == 0) p.dbeta[row0 + r] = nn > 0.f ? d / (p.eps + nn) : 0.f;
        if (kr < 0) continue;
        const float dn = nn > 0.f ? -d * vbeta[r] / ((p.eps + nn) * (p.eps + nn)) : 0.f;
        const float2 xx = *reinterpret_cast<const float2 *>(X + r * LD + 2 * lane);
        const float2 gx = *reinterpret_cast<const float2 *>(U + r * LD + 2 * lane);
        const float g0 = gx.x + 2.f * dn * xx.x, g1 = gx.y + 2.f * dn * xx.y;
        const float xd = group_sum<32>(xx.x * g0 + xx.y * g1);
        const float inv = vinv[r];
        const float2 o = p.phi != 0 ? make_float2(g0, g1) : make_float2((g0 - xx.x * xd) * inv, (g1 - xx.y * xd) * inv);
        *reinterpret_cast<float2 *>(p.dk_out + (bh * (size_t)L + kr) * DD + 2 * lane) = o;
    }
    // under the prefix pair the last key feeds no sample
    if (p.pairing == 0 && t0 + n == L && warp == 0)
        *reinterpret_cast<float2 *>(p.dk_out + (bh * (size_t)L + L - 1) * DD + 2 * lane) = make_float2(0.f, 0.f);
    if (lane == 0) vw[warp] = dl;
    __syncthreads();
    if (tid == 0 && p.dlambda) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NTH / 32; ++w) s += vw[w];
        atomicAdd(&p.dlambda[bh % p.H], s);
    }
}

// ------------------------------------------------------------ launcher
namespace {

size_t al256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool bwd_chunk_covers(const BwdParams &p) {
    return (p.variant == F1 || p.variant == F1A) && p.form == 2 && p.chunk == CC && p.dk == DD && p.dv == DD &&
           p.dtype_bf16;
}

size_t bwd_chunk_ws_bytes(const BwdParams &p) {
    const size_t BH = (size_t)p.B * p.H, nch = (p.L + CC - 1) / CC, units = BH * nch;
    const size_t rows = BH * p.L;
    FwdParams f{};
    f.variant = p.variant; f.B = p.B; f.H = p.H; f.L = p.L; f.dk = DD; f.dv = DD; f.chunk = CC;
    return al256(split_chunk_images_ws_bytes(f))  // the forward's images and g_C
           + al256(units * DD * DD * 4) * 2       // states entering each chunk; G^ leaving each chunk
           + al256(rows * DD * 2)                 // the forward's outputs (unused)
           + al256(BH * DD * DD * 4)              // the forward's final state
           + al256(units * NBND * 4);             // partials of <G^, S_end>
}

int launch_bwd_chunk(const BwdParams &p, void *ws, cudaStream_t s) {
    if (!al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.dout) || !al16(p.dq) || !al16(p.dk_out) ||
        !al16(p.dv_out))
        return 1;  // the vector loads and stores need 16-byte aligned rows
    const int BH = p.B * p.H, nch = (p.L + CC - 1) / CC;
    const size_t units = (size_t)BH * nch, rows = (size_t)BH * p.L;
    uint8_t *base = static_cast<uint8_t *>(ws);
    FwdParams f{};
    f.variant = p.variant; f.form = 2; f.pairing = p.pairing; f.phi = p.phi; f.window = 1;
    f.B = p.B; f.H = p.H; f.L = p.L; f.dk = DD; f.dv = DD; f.chunk = CC; f.eps = p.eps;
    f.q = p.q; f.k = p.k; f.v = p.v; f.beta = p.beta; f.lambda = p.lambda;
    size_t off = 0;
    f.ws = base; f.ws_bytes = split_chunk_images_ws_bytes(f); f.ws_given = 1;
    const uint8_t *img = base;
    const float *gc = reinterpret_cast<const float *>(base + units * IMG_B);
    off += al256(f.ws_bytes);
    float *states = reinterpret_cast<float *>(base + off);
    off += al256(units * DD * DD * 4);
    float *gend = reinterpret_cast<float *>(base + off);
    off += al256(units * DD * DD * 4);
    f.out = base + off;
    off += al256(rows * DD * 2);
    float *fstate = reinterpret_cast<float *>(base + off);
    off += al256((size_t)BH * DD * DD * 4);
    float *bnd = reinterpret_cast<float *>(base + off);
    f.final_state = fstate;
    f.states_out = states;
    const int frc = launch_split_chunk(f, s);
    if (frc != 0) return frc;  // 1: the forward's tensor-core path refused the pointers
    const size_t rbytes = (16 * (size_t)LD + 64 * (size_t)LDC) * sizeof(float) + 2 * (size_t)TILE_B;
    const size_t cbytes = ((size_t)NTILE * TF + NVEC) * sizeof(float);
    static_assert(((size_t)NTILE * TF + NVEC) * sizeof(float) <= 227 * 1024, "shared memory of one block");
    static bool attrs[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaFuncSetAttribute(bwd_rchain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rbytes);
        cudaFuncSetAttribute(bwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cbytes);
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    bwd_rchain_kernel<<<(unsigned)(BH * RQ), NTHR, rbytes, s>>>(p, img, gc, states, fstate, gend, bnd, nch);
    bwd_chunk_kernel<<<(unsigned)units, NTH, cbytes, s>>>(p, states, gend, bnd, nch);
    return cudaGetLastError() == cudaSuccess ? 0 : -7;
}

}  // namespace falcon
