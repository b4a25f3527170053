// k_recurrent.cu -- the recurrent form: token-by-token state update
// ("recurrent: O(d^2) per step", page "Fast Weight Attention：用于持续学习的
// 快速权重注意力", 核心方法 3).
//
// Rows of S are independent (each value channel j only ever reads row j,
// the shared sample x and its own target y_j), so one thread block owns a
// slice of rows of one (b,h) and keeps them in registers for the whole
// sequence: a group of DK/4 lanes holds one row, 4 fp32 per lane.  Token
// tiles of 32 are staged in shared memory (the shifted, normalised samples
// x_t = phi(k_{t-1}) with a halo of window-1 older samples, q_t, the slice
// of y_t, and the per-row step / decay), then every row group runs the tile's
// steps with warp-shuffle reductions only.
#include "common.cuh"
#include "kernels.h"

namespace falcon {

template <typename T, int DK>
__global__ void __launch_bounds__(128) recurrent_kernel(FwdParams p) {
    constexpr int EPT = 4;
    constexpr int LPR = DK / EPT;  // lanes per row
    constexpr int RPW = 32 / LPR;  // rows per warp
    constexpr int RPC = 4 * RPW;   // rows per block
    constexpr int TT = 32;         // tokens per tile
    constexpr int HALO = kMaxWindow - 1;
    __shared__ float xs[(TT + HALO) * DK];
    __shared__ float sqn[TT + HALO];
    __shared__ float qs[TT * DK];
    __shared__ float ys[(TT + HALO) * RPC];
    __shared__ float etas[TT * RPC];
    __shared__ float alphas[TT * RPC];

    const VariantInfo vi = variant_info(p.variant, p.window);
    const int bh = blockIdx.x;
    const int h = bh % p.H;
    const int row0 = blockIdx.y * RPC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp * RPW + lane / LPR;  // row inside the block
    const int sl = lane % LPR;
    const int row = row0 + grp;
    const bool row_ok = row < p.dv;
    const int L = p.L;
    const float lam = p.lambda[h];

    const T *kq = static_cast<const T *>(p.q) + (size_t)bh * L * DK;
    const T *kk = static_cast<const T *>(p.k) + (size_t)bh * L * DK;
    const T *kv = static_cast<const T *>(p.v) + (size_t)bh * L * p.dv;
    const T *kb = static_cast<const T *>(p.beta) + (size_t)bh * L * (vi.per_channel ? p.dv : 1);
    T *ko = static_cast<T *>(p.out) + (size_t)bh * L * p.dv;

    // S_0: the carried state of a continued segment, else zeros
    float S[EPT];
#pragma unroll
    for (int e = 0; e < EPT; ++e)
        S[e] = (p.init_state && row_ok) ? p.init_state[((size_t)bh * p.dv + row) * DK + sl * EPT + e] : 0.f;

    for (int t0 = 0; t0 < L; t0 += TT) {
        const int nt = min(TT, L - t0);
        // halo: the HALO samples before t0 -- at the segment start the carried
        // window (the last window-1 slots), zeros before it
        if (t0 == 0) {
            const int P = vi.window - 1;
            for (int i = threadIdx.x; i < HALO * DK; i += blockDim.x) {
                const int slot = i / DK, m = slot - (HALO - P);  // carried sample m, oldest first
                xs[i] = (p.win && m >= 0) ? p.win[((size_t)bh * P + m) * (DK + p.dv) + i % DK] : 0.f;
            }
            for (int i = threadIdx.x; i < HALO * RPC; i += blockDim.x) {
                const int slot = i / RPC, m = slot - (HALO - P), j = row0 + i % RPC;
                ys[i] = (p.win && m >= 0 && j < p.dv) ? p.win[((size_t)bh * P + m) * (DK + p.dv) + DK + j] : 0.f;
            }
            __syncthreads();
            for (int i = threadIdx.x; i < HALO; i += blockDim.x) {
                float e = 0.f;
                for (int c = 0; c < DK; ++c) e += xs[i * DK + c] * xs[i * DK + c];
                sqn[i] = e;
            }
        } else {
            for (int i = threadIdx.x; i < HALO * DK; i += blockDim.x) xs[i] = xs[TT * DK + i];
            for (int i = threadIdx.x; i < HALO * RPC; i += blockDim.x) ys[i] = ys[TT * RPC + i];
            for (int i = threadIdx.x; i < HALO; i += blockDim.x) sqn[i] = sqn[TT + i];
        }
        __syncthreads();
        // samples, queries, targets: one warp per token
        for (int r = warp; r < nt; r += 4) {
            const int t = t0 + r;
            const int ki = p.pairing == 0 ? t - 1 : t;
            // x of a continued segment's first token is the carried phi(k), as given
            const bool carried = ki < 0 && p.x_prev != nullptr;
            float kv4[DK / 32 > 0 ? DK / 32 : 1];
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < (DK >= 32 ? DK / 32 : 1); ++e) {
                const int c = lane + 32 * e;
                float x = 0.f;
                if (ki >= 0 && c < DK) x = to_f32(kk[(size_t)ki * DK + c]);
                if (carried && c < DK) x = p.x_prev[(size_t)bh * DK + c];
                kv4[e] = x;
                ss += x * x;
            }
            ss = group_sum<32>(ss);
            const float inv = (p.phi == 0 && !carried) ? (ss > 0.f ? rsqrtf(ss) : 0.f) : 1.f;
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < (DK >= 32 ? DK / 32 : 1); ++e) {
                const int c = lane + 32 * e;
                if (c < DK) {
                    const float x = kv4[e] * inv;
                    xs[(HALO + r) * DK + c] = x;
                    qs[r * DK + c] = to_f32(kq[(size_t)t * DK + c]);
                    sq += x * x;
                }
            }
            sq = group_sum<32>(sq);
            if (lane == 0) sqn[HALO + r] = sq;
            for (int j = lane; j < RPC; j += 32)
                ys[(HALO + r) * RPC + j] = (row0 + j < p.dv) ? to_f32(kv[(size_t)t * p.dv + row0 + j]) : 0.f;
        }
        __syncthreads();
        // step sizes and decays per (token, row)
        for (int idx = threadIdx.x; idx < nt * RPC; idx += blockDim.x) {
            const int r = idx / RPC, j = idx % RPC;
            const int t = t0 + r;
            float n = 0.f;
            for (int m = 0; m < vi.window; ++m) n += sqn[HALO + r - m];
            float beta = 0.f;
            if (row0 + j < p.dv)
                beta = to_f32(vi.per_channel ? kb[(size_t)t * p.dv + row0 + j] : kb[t]);
            float eta, alpha;
            step_and_decay(beta, n, p.eps, lam, eta, alpha);
            etas[idx] = eta;
            alphas[idx] = alpha;
        }
        __syncthreads();
        // the sequential steps of this tile, one row per lane group
        for (int r = 0; r < nt; ++r) {
            const int t = t0 + r;
            float res[kMaxWindow];
#pragma unroll
            for (int m = 0; m < kMaxWindow; ++m) {
                res[m] = 0.f;
                if (m < vi.window) {
                    const int sr = HALO + r - (vi.window - 1) + m;
                    float part = 0.f;
#pragma unroll
                    for (int e = 0; e < EPT; ++e) part += S[e] * xs[sr * DK + sl * EPT + e];
                    if (vi.regression) part = group_sum<LPR>(part);
                    const float y = ys[sr * RPC + grp];
                    res[m] = vi.regression ? y - part : y;
                }
            }
            const float eta = etas[r * RPC + grp], alpha = alphas[r * RPC + grp];
            float o = 0.f;
#pragma unroll
            for (int e = 0; e < EPT; ++e) {
                float g = 0.f;
#pragma unroll
                for (int m = 0; m < kMaxWindow; ++m)
                    if (m < vi.window) g += res[m] * xs[(HALO + r - (vi.window - 1) + m) * DK + sl * EPT + e];
                S[e] = alpha * S[e] + eta * g;
                o += S[e] * qs[r * DK + sl * EPT + e];
            }
            o = group_sum<LPR>(o);
            if (sl == 0 && row_ok) ko[(size_t)t * p.dv + row] = from_f32<T>(o);
        }
        __syncthreads();
    }
    if (p.final_state && row_ok) {
        float *fs = p.final_state + ((size_t)bh * p.dv + row) * DK + sl * EPT;
#pragma unroll
        for (int e = 0; e < EPT; ++e) fs[e] = S[e];
    }
}

template <typename T, int DK>
static int launch_recurrent_dk(const FwdParams &p, cudaStream_t s) {
    constexpr int RPC = 4 * (32 / (DK / 4));
    dim3 grid(p.B * p.H, (p.dv + RPC - 1) / RPC);
    recurrent_kernel<T, DK><<<grid, 128, 0, s>>>(p);
    return 0;
}

template <typename T>
int launch_recurrent(const FwdParams &p, cudaStream_t s) {
    switch (p.dk) {
        case 16: return launch_recurrent_dk<T, 16>(p, s);
        case 32: return launch_recurrent_dk<T, 32>(p, s);
        case 64: return launch_recurrent_dk<T, 64>(p, s);
        case 128: return launch_recurrent_dk<T, 128>(p, s);
    }
    return -3;
}

template int launch_recurrent<float>(const FwdParams &, cudaStream_t);
template int launch_recurrent<__nv_bfloat16>(const FwdParams &, cudaStream_t);

}  // namespace falcon
