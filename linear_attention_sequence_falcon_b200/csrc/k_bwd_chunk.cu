// k_bwd_chunk.cu -- the backward pass of the chunk-parallel form for Falcon-1
// and Falcon-1A (bf16 inputs, d_k = d_v = 64, chunk 64): gradients of a loss
// with respect to q, v and the per-token samples x, steps eta and log-decays,
// chunk by chunk in parallel; only fixed-size states cross chunk boundaries.
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
//     E^ = (I + M)^{-T} D_eta U, i.e. by back substitution
//          u_t = U_t - sum_{t'>t} e^{G_{t'-1}-G_t} A[t',t] e^_{t'},  e^_t = eta_t u_t
//          (inner product: e^ = eta o U, u = U)
//     dY = E^ (inner product: eta o U)
//     dQ = D_g dO S0 + K X,                          K = (dO E^T) o Dm
//     dX = K^T Q + D_w E G^ - D_a E^ S0 - (Z + Z^T) X,   Z = (E^ E^T) o Md
//          (inner product: K^T Q + D_w Y G^)
//     u_t = G_t x_t (G_t = dL/dS_t), so per token deta_t = e_t . u_t and
//       dL/dlog alpha_t = F_t - eta_t e_t . u_t, where F_t = <G_t, S_t> obeys
//       F_t = do_t . o_t + F_{t+1} - eta_{t+1} y_{t+1} . u_{t+1} for both
//       families (the transition alpha I - eta x x^T is symmetric); it is
//       summed from the chunk's end, where F = <G^, S_end> + do . o, so no
//       sum runs past a chunk boundary.
// The state entering chunk c comes from the forward's chain (S_c), and
//   G^_c = g_C G^_{c+1} - G^_{c+1} Phi'_c^T + dO_c^T Qt_c
// (Phi' and Qt, the forward's per-chunk operators) runs backwards over the
// chunks of a head in bwd_rchain_kernel; every chunk's gradients then follow
// at once in bwd_chunk_kernel.  The products are 64 x 64 x 64 TF32 warp
// MMAs on fp32 shared-memory tiles (fp32 accumulation).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

constexpr int CC = 64;        // chunk
constexpr int DD = 64;        // d_k = d_v
constexpr int LD = 68;        // fp32 row stride of every shared-memory tile
constexpr int TF = CC * LD;   // floats per tile
constexpr uint32_t TILE_B = 8192;           // one bf16 64 x 64 tile of the forward's image
constexpr uint32_t IMG_B = 4 * TILE_B;      // the forward's per-chunk image
constexpr int NTH = 256;

// C += op(A) op(B) over K = 64 for this warp's 16 x 32 block (rows 16 (w & 3),
// columns 32 (w >> 2)) of a 64 x 64 result; fp32 tiles of row stride LD,
// TF32 products.  op(A)(r, k) = TA ? A[k][r] : A[r][k]; op(B)(k, n) = TB ?
// B[n][k] : B[k][n].
template <bool TA, bool TB>
__device__ __forceinline__ void mma64(const float *A, const float *B, float (&acc)[4][4]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
    const int rb = (warp & 3) * 16, cb = (warp >> 2) * 32;
    auto a_at = [&](int r, int k) { return TA ? A[k * LD + r] : A[r * LD + k]; };
    auto b_at = [&](int k, int n) { return TB ? B[n * LD + k] : B[k * LD + n]; };
#pragma unroll 2
    for (int k0 = 0; k0 < 64; k0 += 8) {
        uint32_t a[4];
        a[0] = tc::f2tf32(a_at(rb + g, k0 + t));
        a[1] = tc::f2tf32(a_at(rb + g + 8, k0 + t));
        a[2] = tc::f2tf32(a_at(rb + g, k0 + t + 4));
        a[3] = tc::f2tf32(a_at(rb + g + 8, k0 + t + 4));
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            uint32_t b[2];
            b[0] = tc::f2tf32(b_at(k0 + t, cb + nt * 8 + g));
            b[1] = tc::f2tf32(b_at(k0 + t + 4, cb + nt * 8 + g));
            tc::mma_tf32(acc[nt], a, b);
        }
    }
}

__device__ __forceinline__ void zero(float (&acc)[4][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
}

// f(row, col, value&) over this warp's accumulator elements
template <typename Fn>
__device__ __forceinline__ void each(float (&acc)[4][4], Fn f) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
    const int rb = (warp & 3) * 16, cb = (warp >> 2) * 32;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) f(rb + g + (e >> 1) * 8, cb + nt * 8 + 2 * t + (e & 1), acc[nt][e]);
}

__device__ __forceinline__ float bf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

// element (r, c) of a 64 x 64 bf16 tile in the 128-byte-swizzled layout the
// forward's image uses (row r at 128 r bytes, 16-byte piece c/8 at c/8 ^ (r & 7))
__device__ __forceinline__ float img_at(const uint8_t *tile, int r, int c) {
    const uint32_t off = tc::sw128(r, c >> 3) + (uint32_t)(c & 7) * 2u;
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tile + off));
}

}  // namespace

// ------------------------------------------------------------ reverse chain
// One block per (b, h): G^ walks the chunks from the last to the first.  At
// chunk c the block stores G^_{c+1} (the gradient of the state the chunk
// leaves) for the per-chunk kernel, then forms
//   G^_c = g_C G^_{c+1} + G^_{c+1} (-Phi'_c^T) + dO_c^T Qt_c
// from the forward's image of the chunk (-Phi'^T and Qt, bf16, swizzled) and
// g_C.  Inner-product family: no -Phi'^T term (the image has none).
__global__ void __launch_bounds__(NTH, 1)
    bwd_rchain_kernel(BwdParams p, const uint8_t *img, const float *gc, float *gend, int nch) {
    extern __shared__ float sm[];
    float *Gh = sm;           // G^ (fp32)
    float *Ph = Gh + TF;      // -Phi'^T of the chunk
    float *Qt = Ph + TF;      // Qt of the chunk
    float *dO = Qt + TF;      // dO of the chunk (rows past L zero)
    const int tid = threadIdx.x;
    const bool reg = p.variant == F1;
    const size_t bh = blockIdx.x;
    const int L = p.L;
    const __nv_bfloat16 *dout = static_cast<const __nv_bfloat16 *>(p.dout) + bh * (size_t)L * DD;
    float acc[4][4];
    // G^ at the end of the sequence: dL/dS_L (or zero)
    for (int e = tid; e < DD * DD; e += NTH) {
        const int j = e / DD, i = e % DD;
        Gh[j * LD + i] = p.dstate ? p.dstate[(bh * DD + j) * DD + i] : 0.f;
    }
    __syncthreads();
    for (int c = nch - 1; c >= 0; --c) {
        const size_t u = bh * nch + c;
        const uint8_t *im = img + u * IMG_B;
        const float g = gc[u];
        float *ge = gend + u * DD * DD;
        // G^_{c+1} out; this chunk's operands in
        for (int e = tid; e < DD * DD; e += NTH) {
            const int r = e / DD, cc = e % DD, t = c * CC + r;
            ge[e] = Gh[r * LD + cc];
            if (reg) Ph[r * LD + cc] = img_at(im, r, cc);
            Qt[r * LD + cc] = img_at(im + TILE_B, r, cc);
            dO[r * LD + cc] = t < L ? bf(dout, (size_t)t * DD + cc) : 0.f;
        }
        __syncthreads();
        zero(acc);
        if (reg) mma64<false, false>(Gh, Ph, acc);  // G^ (-Phi'^T)
        mma64<true, false>(dO, Qt, acc);            // dO^T Qt
        each(acc, [&](int r, int col, float &v) { v += g * Gh[r * LD + col]; });
        __syncthreads();  // every warp has read G^
        each(acc, [&](int r, int col, float &v) { Gh[r * LD + col] = v; });
        __syncthreads();
    }
}

// ------------------------------------------------------------ per-chunk gradients
// One block per (b, h, chunk).  Writes dq, dv (final), dx (before the
// normaliser and feature-map terms), deta = dL/deta, dga = dL/dlog alpha
// (whole: the decay kernel divides by alpha), and dgb = eta y . u.
__global__ void __launch_bounds__(NTH, 1)
    bwd_chunk_kernel(BwdParams p, const float *xs, const float *etas, const float *alphas, const float *states,
                     const float *gend, const float *final_state, int nch, float *dga, float *dgb, float *dgx,
                     float *deta, float *dx) {
    extern __shared__ float sm[];
    float *X = sm, *Q = X + TF, *Y = Q + TF, *dO = Y + TF, *S0 = dO + TF, *Gh = S0 + TF;
    float *MT = Gh + TF;  // e^{G_{t-1}-G_s} A[t,s] (s < t); later Z + Z^T
    float *PD = MT + TF;  // e^{G_t-G_s} P[t,s] (s <= t); later K = (dO E^T) o Dm
    float *E = PD + TF;   // residuals E (regression; inner product: unused)
    float *U = E + TF;    // U, then u
    float *Eh = U + TF;   // E^
    float *vec = Eh + TF;
    float *vG = vec, *veta = vec + 64, *vred = vec + 128;  // vred: [2][64] row partials, then [64] + [64 + 8]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool reg = p.variant == F1;
    const int L = p.L;
    const size_t bh = blockIdx.x / nch;
    const int c = blockIdx.x % nch, t0 = c * CC, n = min(CC, L - t0);
    const size_t row0 = bh * (size_t)L + t0;  // first token of the chunk in [B*H*L]
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(p.q) + row0 * DD;
    const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v) + row0 * DD;
    const __nv_bfloat16 *dout = static_cast<const __nv_bfloat16 *>(p.dout) + row0 * DD;
    const float *x = xs + row0 * DD;
    const float *s0 = states + (bh * nch + c) * DD * DD, *ge = gend + (bh * nch + c) * DD * DD;

    // ---- inputs (rows past the sequence end are zero: no sample, no step)
    for (int e = tid; e < CC * DD; e += NTH) {
        const int r = e / DD, cc = e % DD;
        const bool in = r < n;
        X[r * LD + cc] = in ? x[e] : 0.f;
        Q[r * LD + cc] = in ? bf(q, e) : 0.f;
        Y[r * LD + cc] = in ? bf(v, e) : 0.f;
        dO[r * LD + cc] = in ? bf(dout, e) : 0.f;
        S0[r * LD + cc] = s0[e];
        Gh[r * LD + cc] = ge[e];
    }
    // chunk-local cumulative log decay (one warp) and the steps
    if (warp == 0) {
        float la[2], eta[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int r = lane + 32 * h2;
            const bool in = r < n;
            la[h2] = in ? __logf(alphas[row0 + r]) : 0.f;
            eta[h2] = in ? etas[row0 + r] : 0.f;
        }
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
        veta[lane] = eta[0];
        veta[lane + 32] = eta[1];
    }
    __syncthreads();
    const float GC = vG[CC - 1];
    auto Gm1 = [&](int t) { return t > 0 ? vG[t - 1] : 0.f; };

    float acc[4][4], acc2[4][4];
    // ---- A and P (masked with their decays); U = w~ (X G^^T); R = Y - D_a X S0^T
    zero(acc);
    mma64<false, true>(X, X, acc);
    each(acc, [&](int r, int s, float &val) { MT[r * LD + s] = s < r ? __expf(Gm1(r) - vG[s]) * val : 0.f; });
    zero(acc);
    mma64<false, true>(Q, X, acc);
    each(acc, [&](int r, int s, float &val) { PD[r * LD + s] = s <= r ? __expf(vG[r] - vG[s]) * val : 0.f; });
    zero(acc);
    mma64<false, true>(X, Gh, acc);
    each(acc, [&](int r, int j, float &val) { U[r * LD + j] = __expf(GC - vG[r]) * val; });
    if (reg) {
        zero(acc);
        mma64<false, true>(X, S0, acc);
        each(acc, [&](int r, int j, float &val) { E[r * LD + j] = Y[r * LD + j] - __expf(Gm1(r)) * val; });
    }
    __syncthreads();
    // ---- U += (P o Dm~)^T dO
    zero(acc);
    mma64<true, false>(PD, dO, acc);
    __syncthreads();  // (no tile is written before every warp has read PD and dO)
    each(acc, [&](int r, int j, float &val) { U[r * LD + j] += val; });
    __syncthreads();
    // ---- the two triangular systems, one column per thread: E (forward
    //      substitution, threads 0-63) and E^ / u (back substitution, 64-127)
    const float *et = veta;
    if (reg && tid < 64) {
        const int j = tid;
        for (int t = 1; t < CC; ++t) {
            float s0a = 0.f, s1a = 0.f;
            const float *mrow = MT + t * LD;
            int s = 0;
            for (; s + 1 < t; s += 2) {
                s0a += mrow[s] * et[s] * E[s * LD + j];
                s1a += mrow[s + 1] * et[s + 1] * E[(s + 1) * LD + j];
            }
            if (s < t) s0a += mrow[s] * et[s] * E[s * LD + j];
            E[t * LD + j] -= s0a + s1a;
        }
    } else if (tid >= 64 && tid < 128) {
        const int j = tid - 64;
        for (int t = CC - 1; t >= 0; --t) {
            float uu = U[t * LD + j];
            if (reg) {
                float a0 = 0.f, a1 = 0.f;
                int tp = t + 1;
                for (; tp + 1 < CC; tp += 2) {
                    a0 += MT[tp * LD + t] * Eh[tp * LD + j];
                    a1 += MT[(tp + 1) * LD + t] * Eh[(tp + 1) * LD + j];
                }
                if (tp < CC) a0 += MT[tp * LD + t] * Eh[tp * LD + j];
                uu -= a0 + a1;
            }
            U[t * LD + j] = uu;
            Eh[t * LD + j] = et[t] * uu;
        }
    }
    __syncthreads();
    const float *Ef = reg ? E : Y;  // the residuals (inner product: the targets)
    // ---- O = D_g Q S0^T + (P o Dm) E: do . o per token (row partials of the two column halves)
    zero(acc);
    mma64<false, true>(Q, S0, acc);
    each(acc, [&](int r, int j, float &val) { val *= __expf(vG[r]); });
    {
        // (P o Dm~) diag(eta) E: scale E's rows by eta into Eh's free copy?  E's
        // rows scaled on the fly: (P o Dm~)[r][s] eta_s E[s][j]
        const int g = lane >> 2, tq = lane & 3, rb = (warp & 3) * 16, cb = (warp >> 2) * 32;
#pragma unroll 2
        for (int k0 = 0; k0 < 64; k0 += 8) {
            uint32_t a[4];
            a[0] = tc::f2tf32(PD[(rb + g) * LD + k0 + tq] * et[k0 + tq]);
            a[1] = tc::f2tf32(PD[(rb + g + 8) * LD + k0 + tq] * et[k0 + tq]);
            a[2] = tc::f2tf32(PD[(rb + g) * LD + k0 + tq + 4] * et[k0 + tq + 4]);
            a[3] = tc::f2tf32(PD[(rb + g + 8) * LD + k0 + tq + 4] * et[k0 + tq + 4]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                uint32_t b[2];
                b[0] = tc::f2tf32(Ef[(k0 + tq) * LD + cb + nt * 8 + g]);
                b[1] = tc::f2tf32(Ef[(k0 + tq + 4) * LD + cb + nt * 8 + g]);
                tc::mma_tf32(acc[nt], a, b);
            }
        }
    }
    {
        // row partials of do . o over this warp's 32 columns
        float part[2] = {0.f, 0.f};  // rows rb + g and rb + g + 8
        each(acc, [&](int r, int j, float &val) { part[((r & 15) >> 3)] += dO[r * LD + j] * val; });
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            part[h2] += __shfl_xor_sync(0xffffffffu, part[h2], 1);
            part[h2] += __shfl_xor_sync(0xffffffffu, part[h2], 2);
        }
        if ((lane & 3) == 0) {
            const int rb = (warp & 3) * 16, g = lane >> 2;
            vred[(warp >> 2) * 64 + rb + g] = part[0];
            vred[(warp >> 2) * 64 + rb + g + 8] = part[1];
        }
    }
    // ---- K = (dO E^T) o Dm, over P o Dm (no longer needed once O is formed)
    zero(acc2);
    mma64<false, true>(dO, Ef, acc2);
    __syncthreads();  // every warp has read PD for O
    each(acc2, [&](int r, int s, float &val) { PD[r * LD + s] = s <= r ? __expf(vG[r] - vG[s]) * et[s] * val : 0.f; });
    // ---- per-token terms.  dL/dlog alpha_t = F_t - eta_t e_t . u_t with
    //      F_t = <G_t, S_t> = sum_{t'=t..end} (do . o - eta y . u)_{t'} + eta_t y_t . u_t
    //            + <G^, S_end>
    //      (the boundary term is one inner product per chunk, so the sum never
    //      runs past the chunk end); written as dL/dlog alpha in dga
    float *va = vred + 128, *vx = vred + 192;  // [64] do . o - eta y . u;  [64] the local terms
    if (tid < 64) {
        const int r = tid;
        float yu = 0.f, eu = 0.f;
        for (int j = 0; j < DD; ++j) {
            const float uu = U[r * LD + j];
            yu += Y[r * LD + j] * uu;
            eu += Ef[r * LD + j] * uu;
        }
        const float a = r < n ? vred[r] + vred[64 + r] : 0.f;
        va[r] = r < n ? a - et[r] * yu : 0.f;
        vx[r] = r < n ? et[r] * yu - et[r] * eu : 0.f;  // eta (y - e) . u  (+ eta y . u of F_t)
        if (r < n) {
            deta[row0 + r] = eu;
            dgb[row0 + r] = et[r] * yu;
        }
    }
    {   // <G^, S_end>: S_end is the state entering the next chunk (the final state after the last)
        const float *sn = c + 1 < nch ? states + (bh * nch + c + 1) * DD * DD : final_state + bh * DD * DD;
        float part = 0.f;
        for (int e = tid; e < DD * DD; e += NTH) part += Gh[(e / DD) * LD + e % DD] * sn[e];
        part = group_sum<32>(part);
        if (lane == 0) vx[64 + warp] = part;
    }
    for (int e = tid; e < n * DD; e += NTH) {
        const int r = e / DD, j = e % DD;
        p.dv_out[(row0 + r) * DD + j] = Eh[r * LD + j];
    }
    // ---- Z = (E^ E^T) o Md over the consumed MT (regression)
    if (reg) {
        zero(acc2);
        mma64<false, true>(Eh, E, acc2);
    }
    __syncthreads();  // K is complete; MT is free (the solves are done); per-token terms in place
    if (warp == 0) {
        // reverse (suffix) sum over the chunk of do . o - eta y . u, plus the boundary term
        float bnd = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NTH / 32; ++w2) bnd += vx[64 + w2];
        float s1 = va[63 - lane], s0 = va[31 - lane];  // rows 63-lane and 31-lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y1 = __shfl_up_sync(0xffffffffu, s1, o), y0 = __shfl_up_sync(0xffffffffu, s0, o);
            if (lane >= o) { s1 += y1; s0 += y0; }
        }
        s0 += __shfl_sync(0xffffffffu, s1, 31);  // rows 0-31 also take every row of 32-63
        const int r1 = 63 - lane, r0 = 31 - lane;
        if (r1 < n) dga[row0 + r1] = s1 + bnd + vx[r1];
        if (r0 < n) dga[row0 + r0] = s0 + bnd + vx[r0];
    }
    if (reg)
        each(acc2, [&](int r, int s, float &val) {
            MT[r * LD + s] = s < r ? __expf(Gm1(r) - vG[s]) * et[s] * val : 0.f;
        });
    // ---- dQ = D_g dO S0 + K X
    zero(acc);
    mma64<false, false>(dO, S0, acc);
    each(acc, [&](int r, int i, float &val) { val *= __expf(vG[r]); });
    mma64<false, false>(PD, X, acc);
    each(acc, [&](int r, int i, float &val) {
        if (r < n) p.dq[(row0 + r) * DD + i] = val;
    });
    __syncthreads();  // Z written
    if (reg) {
        // Z + Z^T: mirror the strict lower triangle into the upper one
        for (int e = tid; e < CC * CC; e += NTH) {
            const int r = e / CC, s = e % CC;
            if (s > r) MT[r * LD + s] = MT[s * LD + r];
        }
    }
    __syncthreads();
    // ---- dX = K^T Q + D_w E G^ - D_a E^ S0 - (Z + Z^T) X
    zero(acc);
    mma64<true, false>(PD, Q, acc);
    zero(acc2);
    mma64<false, false>(Ef, Gh, acc2);
    each(acc2, [&](int r, int i, float &val) { val *= __expf(GC - vG[r]) * et[r]; });
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] += acc2[nt][e];
    if (reg) {
        zero(acc2);
        mma64<false, false>(Eh, S0, acc2);
        each(acc2, [&](int r, int i, float &val) { val *= __expf(Gm1(r)); });
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] -= acc2[nt][e];
        zero(acc2);
        mma64<false, false>(MT, X, acc2);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] -= acc2[nt][e];
    }
    each(acc, [&](int r, int i, float &val) {
        if (r < n) dx[(row0 + r) * DD + i] = val;
    });
}

// ------------------------------------------------------------ launcher
namespace {

size_t al256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

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
           + al256(BH * DD * DD * 4);             // the forward's final state
}

int launch_bwd_chunk(const BwdParams &p, void *ws, const float *xs, const float *etas, const float *alphas,
                     float *dga, float *dgb, float *dgx, float *deta, float *dx, cudaStream_t s) {
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
    f.final_state = fstate;
    f.states_out = states;
    const int frc = launch_split_chunk(f, s);
    if (frc != 0) return frc;  // 1: the forward's tensor-core path refused the pointers
    const size_t rbytes = 4 * (size_t)TF * sizeof(float);
    const size_t cbytes = 11 * (size_t)TF * sizeof(float) + 8 * 64 * sizeof(float);
    static bool attrs[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaFuncSetAttribute(bwd_rchain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rbytes);
        cudaFuncSetAttribute(bwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cbytes);
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    bwd_rchain_kernel<<<(unsigned)BH, NTH, rbytes, s>>>(p, img, gc, gend, nch);
    bwd_chunk_kernel<<<(unsigned)units, NTH, cbytes, s>>>(p, xs, etas, alphas, states, gend, fstate, nch, dga, dgb,
                                                          dgx, deta, dx);
    return cudaGetLastError() == cudaSuccess ? 0 : -7;
}

}  // namespace falcon
