// k_span.cu -- chunk-parallel and masked-parallel forms on CUDA cores, fp32.
//
// ("masked-parallel: the recurrence unrolled under a causal mask";
//  "chunk-parallel: parallel inside chunks, recurrent across chunks", page
//  "Fast Weight Attention：用于持续学习的快速权重注意力", 核心方法 3; "only a
//  fixed-size state passes between chunks", page "借鉴40年前的设想！…", 02 (2).)
//
// Both forms solve the same unrolled system.  Inside a span of positions
// [c0, c1) entered with state S0, with G_t = sum_{c0<=r<=t} log alpha_r (per
// value channel for Falcon-2/2A) and the window samples W_t (one sample
// outside Falcon-3/3A):
//   S_t     = e^{G_t} S0 + sum_{s<=t} e^{G_t-G_s} eta_s sum_{i in W_s} r_{s,i} x_i^T
//   r_{t,i} = y_i - e^{G_{t-1}} S0 x_i
//             - sum_{s<t} e^{G_{t-1}-G_s} eta_s sum_{i' in W_s} (x_i'.x_i) r_{s,i'}
//   o_t     = S_t q_t
// (r = y for the inner-product family).  The chunk form walks spans of
// `chunk` tokens and hands S0 on; the masked form never forms a state: it
// sweeps row blocks I and subtracts the contributions of every earlier block
// J through explicit pairwise tiles X_I X_J^T and Q_I X_J^T with the global
// decay e^{Gamma_{t-1}-Gamma_s}, keeping the solved r_J in scratch.
//
// Rows of S (value channels) are independent, so a thread block owns one
// (b,h) and a slice of VS channels; it recomputes the shared Gram tiles.
// Every exponent is a difference Gamma_later - Gamma_earlier <= 0, so no
// factor exceeds 1 whatever the decay.
//
// This is the exact-fp32 path (fp32 inputs) and the reference structure of
// the tensor-core chunk kernel.
#include "common.cuh"
#include "kernels.h"

namespace falcon {

namespace {

constexpr int kThreads = 256;
constexpr int VS = 16;  // value channels per block

// Shared-memory carve-up shared by the host size computation and the kernel.
struct ChunkLayout {
    int C, w, MM, LDX, LDA;
    size_t X, Q, Y, A, P, S0, SX, SQ, ETA, G, R, SQN, total;
    __host__ __device__ ChunkLayout(int C_, int w_, int DK) {
        C = C_; w = w_; MM = C + w - 1; LDX = DK + 1; LDA = MM + 1;
        size_t o = 0;
        X = o; o += (size_t)MM * LDX;
        Q = o; o += (size_t)C * LDX;
        Y = o; o += (size_t)MM * VS;
        A = o; o += (size_t)MM * LDA;
        P = o; o += (size_t)C * LDA;
        S0 = o; o += (size_t)VS * LDX;
        SX = o; o += (size_t)MM * VS;
        SQ = o; o += (size_t)C * VS;
        ETA = o; o += (size_t)C * VS;
        G = o; o += (size_t)C * VS;
        R = o; o += (size_t)C * w * VS;
        SQN = o; o += (size_t)MM;
        total = o;
    }
};

// x_i for sample rows r in [0, nrows): sample index i = i0 + r; prefix pair
// x_i = phi(k_{i-1}), same-step x_i = phi(k_i); zeros for i >= L (rows past
// the end are never read as real samples).  Before the segment: x_0 (prefix
// pair) is the carried phi(k) and the samples i < 0 the carried window of a
// continued segment (zeros at the start of a sequence).  Also y_i for the
// block's channel slice and |x_i|^2.
template <typename T, int DK>
__device__ void load_samples(const FwdParams &p, int bh, const T *kk, const T *kv, int L, int i0, int nrows,
                             int j0, float *X, int LDX, float *Y, float *SQN) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = variant_info(p.variant, p.window).window - 1;
    for (int r = warp; r < nrows; r += kThreads / 32) {
        const int i = i0 + r;
        const int ki = p.pairing == 0 ? i - 1 : i;
        const bool ok = i >= 0 && i < L && ki >= 0;
        // carried samples: the window before the segment, and x_0's phi(k)
        const float *cw = (i < 0 && i >= -P && p.win) ? p.win + ((size_t)bh * P + (i + P)) * (DK + p.dv) : nullptr;
        const bool cx = i == 0 && ki < 0 && p.x_prev != nullptr;
        float ss = 0.f;
        for (int c = lane; c < DK; c += 32) {
            float x = ok ? to_f32(kk[(size_t)ki * DK + c]) : 0.f;
            if (cw) x = cw[c];
            if (cx) x = p.x_prev[(size_t)bh * DK + c];
            X[r * LDX + c] = x;
            ss += x * x;
        }
        ss = group_sum<32>(ss);
        const float inv = (p.phi == 0 && !cw && !cx) ? (ss > 0.f ? rsqrtf(ss) : 0.f) : 1.f;
        float sq = 0.f;
        for (int c = lane; c < DK; c += 32) {
            const float x = X[r * LDX + c] * inv;
            X[r * LDX + c] = x;
            sq += x * x;
        }
        sq = group_sum<32>(sq);
        if (lane == 0) SQN[r] = sq;
        if (lane < VS) {
            const int j = j0 + lane;
            float y = (i >= 0 && i < L && j < p.dv) ? to_f32(kv[(size_t)i * p.dv + j]) : 0.f;
            if (cw && j < p.dv) y = cw[DK + j];
            Y[r * VS + lane] = y;
        }
    }
}

template <typename T, int DK>
__device__ void load_queries(const T *kq, int t0, int n, float *Q, int LDX) {
    for (int idx = threadIdx.x; idx < n * DK; idx += kThreads) {
        const int r = idx / DK, c = idx % DK;
        Q[r * LDX + c] = to_f32(kq[(size_t)(t0 + r) * DK + c]);
    }
}

// C[a][b] = sum_c U[a][c] V[b][c] for a < na, b < nb; each thread a 4x4
// block of C (rows past na / columns past nb read row 0 and are not stored).
template <int DK>
__device__ void small_gemm_nt(const float *U, int ldu, int na, const float *V, int ldv, int nb,
                              float *C, int ldc) {
    const int ta = (na + 3) >> 2, tb = (nb + 3) >> 2;
    for (int idx = threadIdx.x; idx < ta * tb; idx += kThreads) {
        const int a0 = (idx / tb) * 4, b0 = (idx % tb) * 4;
        const float *u[4], *v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            u[i] = U + (a0 + i < na ? a0 + i : 0) * ldu;
            v[i] = V + (b0 + i < nb ? b0 + i : 0) * ldv;
        }
        float acc[4][4] = {};
#pragma unroll 4
        for (int c = 0; c < DK; ++c) {
            float x[4], y[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                x[i] = u[i][c];
                y[i] = v[i][c];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[i][k] = fmaf(x[i], y[k], acc[i][k]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (a0 + i < na && b0 + k < nb) C[(a0 + i) * ldc + b0 + k] = acc[i][k];
    }
}

// eta_{t,j}, log alpha_{t,j} for the n tokens whose windows are sample rows
// [tl, tl+w-1]; beta from global.
template <typename T>
__device__ void steps_and_logdecay(const FwdParams &p, const VariantInfo &vi, const T *kb, int t0, int n,
                                   int j0, float lam, const float *SQN, float *ETA, float *LOGA) {
    for (int idx = threadIdx.x; idx < n * VS; idx += kThreads) {
        const int tl = idx / VS, j = idx % VS;
        const int t = t0 + tl;
        float e = 0.f;
        for (int m = 0; m < vi.window; ++m) e += SQN[tl + m];
        float beta = 0.f;
        if (j0 + j < p.dv) beta = to_f32(vi.per_channel ? kb[(size_t)t * p.dv + j0 + j] : kb[t]);
        float eta, alpha;
        step_and_decay(beta, e, p.eps, lam, eta, alpha);
        ETA[idx] = eta;
        LOGA[idx] = logf(alpha);
    }
}

}  // namespace

// ------------------------------------------------------------------ chunk form

template <typename T, int DK>
__global__ void __launch_bounds__(kThreads) span_chunk_kernel(FwdParams p) {
    extern __shared__ float smem[];
    const VariantInfo vi = variant_info(p.variant, p.window);
    const int w = vi.window;
    const ChunkLayout Lo(p.chunk, w, DK);
    float *X = smem + Lo.X, *Q = smem + Lo.Q, *Y = smem + Lo.Y, *A = smem + Lo.A, *P = smem + Lo.P;
    float *S0 = smem + Lo.S0, *SX = smem + Lo.SX, *SQ = smem + Lo.SQ, *ETA = smem + Lo.ETA;
    float *G = smem + Lo.G, *R = smem + Lo.R, *SQN = smem + Lo.SQN;
    const int LDX = Lo.LDX, LDA = Lo.LDA;

    const int bh = blockIdx.x, h = bh % p.H;
    const int j0 = blockIdx.y * VS;
    const int L = p.L, dv = p.dv;
    const float lam = p.lambda[h];
    const T *kq = static_cast<const T *>(p.q) + (size_t)bh * L * DK;
    const T *kk = static_cast<const T *>(p.k) + (size_t)bh * L * DK;
    const T *kv = static_cast<const T *>(p.v) + (size_t)bh * L * dv;
    const T *kb = static_cast<const T *>(p.beta) + (size_t)bh * L * (vi.per_channel ? dv : 1);
    T *ko = static_cast<T *>(p.out) + (size_t)bh * L * dv;

    // S0: the carried state of a continued segment, else zeros
    for (int idx = threadIdx.x; idx < VS * LDX; idx += kThreads) {
        const int j = idx / LDX, c = idx % LDX;
        S0[idx] = (p.init_state && c < DK && j0 + j < dv) ? p.init_state[((size_t)bh * dv + j0 + j) * DK + c] : 0.f;
    }

    for (int c0 = 0; c0 < L; c0 += p.chunk) {
        const int n = min(p.chunk, L - c0);
        const int ns = n + w - 1;
        __syncthreads();
        load_samples<T, DK>(p, bh, kk, kv, L, c0 - (w - 1), ns, j0, X, LDX, Y, SQN);
        load_queries<T, DK>(kq, c0, n, Q, LDX);
        __syncthreads();
        steps_and_logdecay<T>(p, vi, kb, c0, n, j0, lam, SQN, ETA, G);
        if (vi.regression) small_gemm_nt<DK>(X, LDX, ns, X, LDX, ns, A, LDA);
        small_gemm_nt<DK>(Q, LDX, n, X, LDX, ns, P, LDA);
        if (vi.regression) small_gemm_nt<DK>(X, LDX, ns, S0, LDX, VS, SX, VS);
        small_gemm_nt<DK>(Q, LDX, n, S0, LDX, VS, SQ, VS);
        __syncthreads();
        // cumulative log decay inside the chunk
        if (threadIdx.x < VS) {
            float acc = 0.f;
            for (int tl = 0; tl < n; ++tl) {
                acc += G[tl * VS + threadIdx.x];
                G[tl * VS + threadIdx.x] = acc;
            }
        }
        __syncthreads();
        // right-hand sides
        for (int idx = threadIdx.x; idx < n * w * VS; idx += kThreads) {
            const int tl = idx / (w * VS), m = (idx / VS) % w, j = idx % VS;
            float r = Y[(tl + m) * VS + j];
            if (vi.regression) {
                const float gp = tl > 0 ? G[(tl - 1) * VS + j] : 0.f;
                r -= expf(gp) * SX[(tl + m) * VS + j];
            }
            R[idx] = r;
        }
        // forward substitution, column by column
        if (vi.regression) {
            for (int s = 0; s + 1 < n; ++s) {
                __syncthreads();
                const int cnt = (n - 1 - s) * w * VS;
                for (int idx = threadIdx.x; idx < cnt; idx += kThreads) {
                    const int tl = s + 1 + idx / (w * VS), m = (idx / VS) % w, j = idx % VS;
                    const float coef = expf(G[(tl - 1) * VS + j] - G[s * VS + j]) * ETA[s * VS + j];
                    float acc = 0.f;
                    for (int m2 = 0; m2 < w; ++m2) acc += A[(tl + m) * LDA + s + m2] * R[(s * w + m2) * VS + j];
                    R[(tl * w + m) * VS + j] -= coef * acc;
                }
            }
        }
        __syncthreads();
        // outputs o_t = S_t q_t
        for (int idx = threadIdx.x; idx < n * VS; idx += kThreads) {
            const int tl = idx / VS, j = idx % VS;
            const float gt = G[tl * VS + j];
            float o = expf(gt) * SQ[idx];
            for (int s = 0; s <= tl; ++s) {
                const float coef = expf(gt - G[s * VS + j]) * ETA[s * VS + j];
                float acc = 0.f;
                for (int m = 0; m < w; ++m) acc += P[tl * LDA + s + m] * R[(s * w + m) * VS + j];
                o += coef * acc;
            }
            if (j0 + j < dv) ko[(size_t)(c0 + tl) * dv + j0 + j] = from_f32<T>(o);
        }
        // state hand-off S0 <- S_{c1-1}; the weights e^{G_end - G_s} eta_s once per
        // token (SX is free once the right-hand sides are formed)
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * VS; idx += kThreads)
            SX[idx] = expf(G[(n - 1) * VS + idx % VS] - G[idx]) * ETA[idx];
        __syncthreads();
        for (int idx = threadIdx.x; idx < VS * DK; idx += kThreads) {
            const int j = idx / DK, c = idx % DK;
            const float ge = G[(n - 1) * VS + j];
            float s = expf(ge) * S0[j * LDX + c];
            for (int sl = 0; sl < n; ++sl) {
                float acc = 0.f;
                for (int m = 0; m < w; ++m) acc += R[(sl * w + m) * VS + j] * X[(sl + m) * LDX + c];
                s += SX[sl * VS + j] * acc;
            }
            S0[j * LDX + c] = s;
        }
    }
    __syncthreads();
    if (p.final_state) {
        for (int idx = threadIdx.x; idx < VS * DK; idx += kThreads) {
            const int j = idx / DK, c = idx % DK;
            if (j0 + j < dv) p.final_state[((size_t)bh * dv + j0 + j) * DK + c] = S0[j * LDX + c];
        }
    }
}

// ------------------------------------------------------------------ masked form

namespace {
struct MaskedLayout {
    int C, w, MM, LDX, LDA;
    size_t XI, QI, XJ, RI, RJ, ETAI, GAMI, ETAJ, GAMJ, A, P, O, S, Y, SQN, SQNJ, YJ, GPREV, GLAST, total;
    __host__ __device__ MaskedLayout(int C_, int w_, int DK) {
        C = C_; w = w_; MM = C + w - 1; LDX = DK + 1; LDA = MM + 1;
        size_t o = 0;
        XI = o; o += (size_t)MM * LDX;
        QI = o; o += (size_t)C * LDX;
        XJ = o; o += (size_t)MM * LDX;
        RI = o; o += (size_t)C * w * VS;
        RJ = o; o += (size_t)C * w * VS;
        ETAI = o; o += (size_t)C * VS;
        GAMI = o; o += (size_t)C * VS;
        ETAJ = o; o += (size_t)C * VS;
        GAMJ = o; o += (size_t)C * VS;
        A = o; o += (size_t)MM * LDA;
        P = o; o += (size_t)C * LDA;
        O = o; o += (size_t)C * VS;
        S = o; o += (size_t)VS * LDX;
        Y = o; o += (size_t)MM * VS;
        SQN = o; o += (size_t)MM;
        SQNJ = o; o += (size_t)MM;
        YJ = o; o += (size_t)MM * VS;
        GPREV = o; o += VS;
        GLAST = o; o += VS;
        total = o;
    }
};
}  // namespace

size_t masked_ws_r_floats(const FwdParams &p) {
    const VariantInfo vi = variant_info(p.variant, p.window);
    return (size_t)p.B * p.H * p.L * vi.window * p.dv;
}
size_t masked_ws_eg_floats(const FwdParams &p) { return (size_t)p.B * p.H * p.L * p.dv; }

template <typename T, int DK>
__global__ void __launch_bounds__(kThreads) span_masked_kernel(FwdParams p, int C) {
    extern __shared__ float smem[];
    const VariantInfo vi = variant_info(p.variant, p.window);
    const int w = vi.window;
    const MaskedLayout Lo(C, w, DK);
    float *XI = smem + Lo.XI, *QI = smem + Lo.QI, *XJ = smem + Lo.XJ, *RI = smem + Lo.RI, *RJ = smem + Lo.RJ;
    float *ETAI = smem + Lo.ETAI, *GAMI = smem + Lo.GAMI, *ETAJ = smem + Lo.ETAJ, *GAMJ = smem + Lo.GAMJ;
    float *A = smem + Lo.A, *P = smem + Lo.P, *O = smem + Lo.O, *S = smem + Lo.S, *Y = smem + Lo.Y;
    float *SQN = smem + Lo.SQN, *SQNJ = smem + Lo.SQNJ, *YJ = smem + Lo.YJ;
    float *GPREV = smem + Lo.GPREV, *GLAST = smem + Lo.GLAST;
    const int LDX = Lo.LDX, LDA = Lo.LDA;

    const int bh = blockIdx.x, h = bh % p.H;
    const int j0 = blockIdx.y * VS;
    const int L = p.L, dv = p.dv;
    const float lam = p.lambda[h];
    const T *kq = static_cast<const T *>(p.q) + (size_t)bh * L * DK;
    const T *kk = static_cast<const T *>(p.k) + (size_t)bh * L * DK;
    const T *kv = static_cast<const T *>(p.v) + (size_t)bh * L * dv;
    const T *kb = static_cast<const T *>(p.beta) + (size_t)bh * L * (vi.per_channel ? dv : 1);
    T *ko = static_cast<T *>(p.out) + (size_t)bh * L * dv;
    // scratch rows of this (b,h); channel j of token t at [t*dv + j0 + j]
    float *wr = p.ws_r + (size_t)bh * L * w * dv;
    float *weta = p.ws_eta + (size_t)bh * L * dv;
    float *wgam = p.ws_gam + (size_t)bh * L * dv;

    // pass 1: eta and the global cumulative log decay Gamma for every token
    if (threadIdx.x < VS) GPREV[threadIdx.x] = 0.f;
    for (int c0 = 0; c0 < L; c0 += C) {
        const int n = min(C, L - c0);
        __syncthreads();
        load_samples<T, DK>(p, bh, kk, kv, L, c0 - (w - 1), n + w - 1, j0, XI, LDX, Y, SQN);
        __syncthreads();
        steps_and_logdecay<T>(p, vi, kb, c0, n, j0, lam, SQN, ETAI, GAMI);
        __syncthreads();
        if (threadIdx.x < VS) {
            float acc = GPREV[threadIdx.x];
            for (int tl = 0; tl < n; ++tl) {
                acc += GAMI[tl * VS + threadIdx.x];
                GAMI[tl * VS + threadIdx.x] = acc;
            }
            GPREV[threadIdx.x] = acc;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * VS; idx += kThreads) {
            const int tl = idx / VS, j = idx % VS;
            if (j0 + j < dv) {
                weta[(size_t)(c0 + tl) * dv + j0 + j] = ETAI[idx];
                wgam[(size_t)(c0 + tl) * dv + j0 + j] = GAMI[idx];
            }
        }
    }
    __syncthreads();
    if (threadIdx.x < VS) GLAST[threadIdx.x] = GPREV[threadIdx.x];
    for (int idx = threadIdx.x; idx < VS * LDX; idx += kThreads) S[idx] = 0.f;

    // pass 2: row blocks in causal order
    for (int c0 = 0; c0 < L; c0 += C) {
        const int n = min(C, L - c0);
        const int ns = n + w - 1;
        __syncthreads();
        load_samples<T, DK>(p, bh, kk, kv, L, c0 - (w - 1), ns, j0, XI, LDX, Y, SQN);
        load_queries<T, DK>(kq, c0, n, QI, LDX);
        for (int idx = threadIdx.x; idx < n * VS; idx += kThreads) {
            const int tl = idx / VS, j = idx % VS;
            const bool ok = j0 + j < dv;
            ETAI[idx] = ok ? weta[(size_t)(c0 + tl) * dv + j0 + j] : 0.f;
            GAMI[idx] = ok ? wgam[(size_t)(c0 + tl) * dv + j0 + j] : 0.f;
            O[idx] = 0.f;
        }
        if (threadIdx.x < VS)
            GPREV[threadIdx.x] = (c0 > 0 && j0 + threadIdx.x < dv) ? wgam[(size_t)(c0 - 1) * dv + j0 + threadIdx.x] : 0.f;
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * w * VS; idx += kThreads) {
            const int tl = idx / (w * VS), m = (idx / VS) % w, j = idx % VS;
            RI[idx] = Y[(tl + m) * VS + j];
        }
        // earlier blocks J: explicit pairwise tiles
        for (int cj = 0; cj < c0; cj += C) {
            const int nj = C;  // earlier blocks are always full
            __syncthreads();
            load_samples<T, DK>(p, bh, kk, kv, L, cj - (w - 1), nj + w - 1, j0, XJ, LDX, YJ, SQNJ);
            // e^{Gamma_a - Gamma_s} for a in block I and s in block J < I splits at
            // Gamma_{c0-1}, the end of the previous block, into two factors <= 1:
            // ETAJ carries e^{Gamma_{c0-1} - Gamma_s} eta_s, the rows their own factor
            for (int idx = threadIdx.x; idx < nj * VS; idx += kThreads) {
                const int tl = idx / VS, j = idx % VS;
                const bool ok = j0 + j < dv;
                ETAJ[idx] = ok ? weta[(size_t)(cj + tl) * dv + j0 + j] *
                                     expf(GPREV[j] - wgam[(size_t)(cj + tl) * dv + j0 + j])
                               : 0.f;
            }
            for (int idx = threadIdx.x; idx < nj * w * VS; idx += kThreads) {
                const int tl = idx / (w * VS), m = (idx / VS) % w, j = idx % VS;
                RJ[idx] = (j0 + j < dv) ? wr[((size_t)(cj + tl) * w + m) * dv + j0 + j] : 0.f;
            }
            __syncthreads();
            if (vi.regression) small_gemm_nt<DK>(XI, LDX, ns, XJ, LDX, nj + w - 1, A, LDA);
            small_gemm_nt<DK>(QI, LDX, n, XJ, LDX, nj + w - 1, P, LDA);
            __syncthreads();
            if (vi.regression) {
                for (int idx = threadIdx.x; idx < n * w * VS; idx += kThreads) {
                    const int tl = idx / (w * VS), m = (idx / VS) % w, j = idx % VS;
                    const float gp = tl > 0 ? GAMI[(tl - 1) * VS + j] : GPREV[j];
                    float acc = 0.f;
                    for (int s = 0; s < nj; ++s) {
                        float a2 = 0.f;
                        for (int m2 = 0; m2 < w; ++m2) a2 += A[(tl + m) * LDA + s + m2] * RJ[(s * w + m2) * VS + j];
                        acc += ETAJ[s * VS + j] * a2;
                    }
                    RI[idx] -= expf(gp - GPREV[j]) * acc;
                }
            }
            for (int idx = threadIdx.x; idx < n * VS; idx += kThreads) {
                const int tl = idx / VS, j = idx % VS;
                const float gt = GAMI[idx];
                float acc = 0.f;
                for (int s = 0; s < nj; ++s) {
                    float a2 = 0.f;
                    for (int m2 = 0; m2 < w; ++m2) a2 += P[tl * LDA + s + m2] * RJ[(s * w + m2) * VS + j];
                    acc += ETAJ[s * VS + j] * a2;
                }
                O[idx] += expf(gt - GPREV[j]) * acc;
            }
        }
        // the diagonal block
        __syncthreads();
        if (vi.regression) small_gemm_nt<DK>(XI, LDX, ns, XI, LDX, ns, A, LDA);
        small_gemm_nt<DK>(QI, LDX, n, XI, LDX, ns, P, LDA);
        if (vi.regression) {
            for (int s = 0; s + 1 < n; ++s) {
                __syncthreads();
                const int cnt = (n - 1 - s) * w * VS;
                for (int idx = threadIdx.x; idx < cnt; idx += kThreads) {
                    const int tl = s + 1 + idx / (w * VS), m = (idx / VS) % w, j = idx % VS;
                    const float coef = expf(GAMI[(tl - 1) * VS + j] - GAMI[s * VS + j]) * ETAI[s * VS + j];
                    float acc = 0.f;
                    for (int m2 = 0; m2 < w; ++m2) acc += A[(tl + m) * LDA + s + m2] * RI[(s * w + m2) * VS + j];
                    RI[(tl * w + m) * VS + j] -= coef * acc;
                }
            }
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * VS; idx += kThreads) {
            const int tl = idx / VS, j = idx % VS;
            const float gt = GAMI[idx];
            float o = O[idx];
            for (int s = 0; s <= tl; ++s) {
                const float coef = expf(gt - GAMI[s * VS + j]) * ETAI[s * VS + j];
                float acc = 0.f;
                for (int m = 0; m < w; ++m) acc += P[tl * LDA + s + m] * RI[(s * w + m) * VS + j];
                o += coef * acc;
            }
            if (j0 + j < dv) ko[(size_t)(c0 + tl) * dv + j0 + j] = from_f32<T>(o);
        }
        for (int idx = threadIdx.x; idx < n * w * VS; idx += kThreads) {
            const int tl = idx / (w * VS), m = (idx / VS) % w, j = idx % VS;
            if (j0 + j < dv) wr[((size_t)(c0 + tl) * w + m) * dv + j0 + j] = RI[idx];
        }
        // the final state's weights e^{Gamma_L - Gamma_s} eta_s, once per token (GAMJ is free here)
        for (int idx = threadIdx.x; idx < n * VS; idx += kThreads)
            GAMJ[idx] = expf(GLAST[idx % VS] - GAMI[idx]) * ETAI[idx];
        __syncthreads();
        for (int idx = threadIdx.x; idx < VS * DK; idx += kThreads) {
            const int j = idx / DK, c = idx % DK;
            float s = 0.f;
            for (int sl = 0; sl < n; ++sl) {
                float acc = 0.f;
                for (int m = 0; m < w; ++m) acc += RI[(sl * w + m) * VS + j] * XI[(sl + m) * LDX + c];
                s += GAMJ[sl * VS + j] * acc;
            }
            S[j * LDX + c] += s;
        }
    }
    __syncthreads();
    if (p.final_state) {
        for (int idx = threadIdx.x; idx < VS * DK; idx += kThreads) {
            const int j = idx / DK, c = idx % DK;
            if (j0 + j < dv) p.final_state[((size_t)bh * dv + j0 + j) * DK + c] = S[j * LDX + c];
        }
    }
}

// ------------------------------------------------------------------ launchers

template <typename T, int DK>
static int launch_chunk_dk(const FwdParams &p, cudaStream_t s) {
    const VariantInfo vi = variant_info(p.variant, p.window);
    const ChunkLayout Lo(p.chunk, vi.window, DK);
    const size_t bytes = Lo.total * sizeof(float);
    if (bytes > 227 * 1024) return -4;
    cudaFuncSetAttribute(span_chunk_kernel<T, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    dim3 grid(p.B * p.H, (p.dv + VS - 1) / VS);
    span_chunk_kernel<T, DK><<<grid, kThreads, bytes, s>>>(p);
    return 0;
}

template <typename T>
int launch_span_chunk(const FwdParams &p, cudaStream_t s) {
    switch (p.dk) {
        case 16: return launch_chunk_dk<T, 16>(p, s);
        case 32: return launch_chunk_dk<T, 32>(p, s);
        case 64: return launch_chunk_dk<T, 64>(p, s);
        case 128: return launch_chunk_dk<T, 128>(p, s);
    }
    return -3;
}

template <typename T, int DK>
static int launch_masked_dk(const FwdParams &p, cudaStream_t s) {
    const VariantInfo vi = variant_info(p.variant, p.window);
    int C = 64;
    size_t bytes = MaskedLayout(C, vi.window, DK).total * sizeof(float);
    while (bytes > 200 * 1024 && C > 16) {
        C /= 2;
        bytes = MaskedLayout(C, vi.window, DK).total * sizeof(float);
    }
    cudaFuncSetAttribute(span_masked_kernel<T, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    dim3 grid(p.B * p.H, (p.dv + VS - 1) / VS);
    span_masked_kernel<T, DK><<<grid, kThreads, bytes, s>>>(p, C);
    return 0;
}

template <typename T>
int launch_span_masked(const FwdParams &p, cudaStream_t s) {
    switch (p.dk) {
        case 16: return launch_masked_dk<T, 16>(p, s);
        case 32: return launch_masked_dk<T, 32>(p, s);
        case 64: return launch_masked_dk<T, 64>(p, s);
        case 128: return launch_masked_dk<T, 128>(p, s);
    }
    return -3;
}

template int launch_span_chunk<float>(const FwdParams &, cudaStream_t);
template int launch_span_chunk<__nv_bfloat16>(const FwdParams &, cudaStream_t);
template int launch_span_masked<float>(const FwdParams &, cudaStream_t);
template int launch_span_masked<__nv_bfloat16>(const FwdParams &, cudaStream_t);

}  // namespace falcon
