// k_chunk_seq.cu -- chunk-parallel forward of Falcon-1 and Falcon-1A (bf16
// inputs, d_k = d_v = d in {32, 64, 128}) for the chunk lengths the fused
// kernel (d = 64, chunk 64) does not take: 16, 32, 64 and 128 (chunk 128 for
// d <= 64), on the tensor cores (TF32 warp MMAs on fp32 shared-memory tiles,
// fp32 accumulation).
//
// The chunk length is the pages' latency/memory knob ("start at chunk = 512
// and measure the curve at 128/256/512/1024", page "Fast Weight Attention：
// 用于持续学习的快速权重注意力", 工程落地); the chunk form is "parallel inside
// chunks, recurrent across chunks" (same page, 核心方法 3).  Chunk 64 runs the
// split two-kernel path (k_chunk_split.cu); the other lengths run here, one
// block per (b, h) walking its chunks.  A chunk of n <= C tokens entered with
// state S0, chunk-local G_t = sum_{r<=t} log alpha_r:
//   A = X X^T, P = Q X^T                              (C x C, K = 64)
//   M[t,s] = e^{G_{t-1}-G_s} eta_s A[t,s]  (s < t)     (regression only)
//   E = (I + M)^{-1} (Y - D_a X S0^T)                  (inner product: E = Y)
//   O = D_g Q S0^T + (P o Dm) E,  Dm[t,s] = e^{G_t-G_s} eta_s (s <= t)
//   S_end = e^{G_C} S0 + E^T D_w X,  w_s = e^{G_C-G_s} eta_s
// (the masked-parallel relation restricted to the chunk, with S0 carried).
// Every decay factor is one exponential of a difference of cumulative logs,
// hence <= 1.  The triangular system is solved by forward substitution, one
// value channel per thread.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

constexpr int NTHS = 256;

template <int C, int DD>
struct SeqLayout {
    static constexpr int LDX = DD + 4;  // fp32 row stride of the C x d and d x d tiles
    static constexpr int LDM = C + 4;   // row stride of the C x C tile
    // X, Q, E (C x d); MP: P o Dm in the lower triangle (diagonal included)
    // and M transposed in the strict upper triangle (M[t][s] at [s][t]); S0
    // (d x d); per-token vectors
    static constexpr size_t X = 0, Q = X + (size_t)C * LDX, E = Q + (size_t)C * LDX, MP = E + (size_t)C * LDX,
                            S0 = MP + (size_t)C * LDM, VEC = S0 + (size_t)DD * LDX, total = VEC + 4 * C + 64;
    static constexpr size_t bytes = total * sizeof(float);
};

// c (16 x 8 at rows r0, columns n0) += sum_{k < K} op(A)(r, k) op(B)(k, n),
// op(A)(r, k) = TA ? A[k][r] : A[r][k], op(B)(k, n) = TB ? B[n][k] : B[k][n]
template <bool TA, bool TB>
__device__ __forceinline__ void mma16x8(const float *A, int lda, const float *B, int ldb, int r0, int n0, int K,
                                        float (&c)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    auto a_at = [&](int r, int k) { return TA ? A[k * lda + r] : A[r * lda + k]; };
    auto b_at = [&](int k, int n) { return TB ? B[n * ldb + k] : B[k * ldb + n]; };
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t a[4], b[2];
        a[0] = tc::f2tf32(a_at(r0 + g, k0 + t));
        a[1] = tc::f2tf32(a_at(r0 + g + 8, k0 + t));
        a[2] = tc::f2tf32(a_at(r0 + g, k0 + t + 4));
        a[3] = tc::f2tf32(a_at(r0 + g + 8, k0 + t + 4));
        b[0] = tc::f2tf32(b_at(k0 + t, n0 + g));
        b[1] = tc::f2tf32(b_at(k0 + t + 4, n0 + g));
        tc::mma_tf32(c, a, b);
    }
}

// f(row, col, value) for the four elements of this lane in a 16 x 8 tile
template <typename Fn>
__device__ __forceinline__ void each16x8(int r0, int n0, const float (&c)[4], Fn f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    f(r0 + g, n0 + 2 * t, c[0]);
    f(r0 + g, n0 + 2 * t + 1, c[1]);
    f(r0 + g + 8, n0 + 2 * t, c[2]);
    f(r0 + g + 8, n0 + 2 * t + 1, c[3]);
}

}  // namespace

template <int C, int DD>
__global__ void __launch_bounds__(NTHS, 1) seq_chunk_kernel(FwdParams p) {
    using Lo = SeqLayout<C, DD>;
    constexpr int LDM = Lo::LDM, LDX = Lo::LDX, EPL = DD / 32;  // elements of a row per lane
    extern __shared__ float sm[];
    float *X = sm + Lo::X, *Q = sm + Lo::Q, *E = sm + Lo::E, *MP = sm + Lo::MP, *S0 = sm + Lo::S0;
    float *vG = sm + Lo::VEC, *veta = vG + C, *vw = veta + C, *vla = vw + C, *vsc = vla + C;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool reg = p.variant == F1;
    const int L = p.L;
    const size_t bh = blockIdx.x;
    const float lam = p.lambda[bh % p.H];
    const __nv_bfloat16 *kq = static_cast<const __nv_bfloat16 *>(p.q) + bh * (size_t)L * DD;
    const __nv_bfloat16 *kk = static_cast<const __nv_bfloat16 *>(p.k) + bh * (size_t)L * DD;
    const __nv_bfloat16 *kv = static_cast<const __nv_bfloat16 *>(p.v) + bh * (size_t)L * DD;
    const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(p.beta) + bh * (size_t)L;
    __nv_bfloat16 *ko = static_cast<__nv_bfloat16 *>(p.out) + bh * (size_t)L * DD;

    // S0: the carried state of a continued segment, else zeros
    for (int e = tid; e < DD * DD; e += NTHS) {
        const int j = e / DD, i = e % DD;
        S0[j * LDX + i] = p.init_state ? p.init_state[bh * DD * DD + e] : 0.f;
    }
    for (int c0 = 0; c0 < L; c0 += C) {
        const int n = min(C, L - c0);
        __syncthreads();
        // ---- samples x_t = phi(k_{t-1}) (prefix pair; phi(k_t) same-step), one warp per row
        for (int r = warp; r < C; r += NTHS / 32) {
            const int t = c0 + r, ki = p.pairing == 0 ? t - 1 : t;
            const bool carried = r < n && ki < 0 && p.x_prev != nullptr;  // x of a continued segment's first token
            const bool in = r < n;
            float xv[EPL];
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                const int cc = lane + 32 * e;
                xv[e] = carried ? p.x_prev[bh * DD + cc]
                                : (in && ki >= 0 ? __bfloat162float(kk[(size_t)ki * DD + cc]) : 0.f);
                ss += xv[e] * xv[e];
            }
            ss = group_sum<32>(ss);
            const float inv = (p.phi != 0 || carried) ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                const int cc = lane + 32 * e;
                const float x = xv[e] * inv;
                sq += x * x;
                X[r * LDX + cc] = x;
                Q[r * LDX + cc] = in ? __bfloat162float(kq[(size_t)t * DD + cc]) : 0.f;
                E[r * LDX + cc] = in ? __bfloat162float(kv[(size_t)t * DD + cc]) : 0.f;
            }
            sq = group_sum<32>(sq);
            if (lane == 0) {
                float eta = 0.f, alpha = 1.f;
                if (in) step_and_decay(__bfloat162float(kb[t]), sq, p.eps, lam, eta, alpha);
                veta[r] = eta;
                vla[r] = __logf(alpha);
            }
        }
        __syncthreads();
        // ---- cumulative log decay (one warp, C / 32 passes with a carry)
        if (warp == 0) {
            float carry = 0.f;
            for (int b0 = 0; b0 < C; b0 += 32) {
                float v = lane < C - b0 ? vla[b0 + lane] : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v += y;
                }
                if (lane < C - b0) vG[b0 + lane] = v + carry;
                carry += __shfl_sync(0xffffffffu, v, 31);
            }
            if (lane == 0) vsc[0] = carry;  // G_C
        }
        __syncthreads();
        const float GC = vsc[0];
        auto Gm1 = [&](int t) { return t > 0 ? vG[t - 1] : 0.f; };
        // ---- P o Dm (lower triangle) and M^T (strict upper triangle) in MP;
        //      R = Y - D_a X S0^T in place over Y (regression)
        {
            constexpr int NPT = (C / 16) * (C / 8);  // 16 x 8 tiles of a C x C product
            for (int tt = warp; tt < NPT; tt += NTHS / 32) {
                const int r0 = (tt / (C / 8)) * 16, n0 = (tt % (C / 8)) * 8;
                if (n0 > r0 + 15) continue;  // strictly above the diagonal: masked out
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                mma16x8<false, true>(Q, LDX, X, LDX, r0, n0, DD, c);
                each16x8(r0, n0, c, [&](int t, int s, float v) {
                    if (s <= t) MP[t * LDM + s] = __expf(vG[t] - vG[s]) * veta[s] * v;
                });
                if (reg) {
                    float a[4] = {0.f, 0.f, 0.f, 0.f};
                    mma16x8<false, true>(X, LDX, X, LDX, r0, n0, DD, a);
                    each16x8(r0, n0, a, [&](int t, int s, float v) {
                        if (s < t) MP[s * LDM + t] = __expf(Gm1(t) - vG[s]) * veta[s] * v;
                    });
                }
            }
            if (reg) {
                constexpr int NXT = (C / 16) * (DD / 8);
                for (int tt = warp; tt < NXT; tt += NTHS / 32) {
                    const int r0 = (tt / (DD / 8)) * 16, n0 = (tt % (DD / 8)) * 8;
                    float c[4] = {0.f, 0.f, 0.f, 0.f};
                    mma16x8<false, true>(X, LDX, S0, LDX, r0, n0, DD, c);
                    // E holds Y; every element read and written by this lane only
                    each16x8(r0, n0, c, [&](int t, int j, float v) { E[t * LDX + j] -= __expf(Gm1(t)) * v; });
                }
            }
        }
        __syncthreads();
        // ---- forward substitution for E, one value channel per thread
        if (reg && tid < DD) {
            const int j = tid;
            for (int t = 1; t < n; ++t) {
                float a0 = 0.f, a1 = 0.f;
                int s = 0;
                for (; s + 1 < t; s += 2) {
                    a0 += MP[s * LDM + t] * E[s * LDX + j];
                    a1 += MP[(s + 1) * LDM + t] * E[(s + 1) * LDX + j];
                }
                if (s < t) a0 += MP[s * LDM + t] * E[s * LDX + j];
                E[t * LDX + j] -= a0 + a1;
            }
        }
        __syncthreads();
        // ---- O = D_g Q S0^T + (P o Dm) E; then the state's weights over E
        {
            constexpr int NOT = (C / 16) * (DD / 8);
            for (int tt = warp; tt < NOT; tt += NTHS / 32) {
                const int r0 = (tt / (DD / 8)) * 16, n0 = (tt % (DD / 8)) * 8;
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                mma16x8<false, true>(Q, LDX, S0, LDX, r0, n0, DD, c);
                const int lane_g = lane >> 2;
#pragma unroll
                for (int e = 0; e < 4; ++e) c[e] *= __expf(vG[r0 + lane_g + (e >> 1) * 8]);
                {   // (P o Dm) E over s <= t: MP's strict upper triangle holds M^T, so mask it
                    const int g = lane >> 2, t4 = lane & 3;
                    for (int k0 = 0; k0 < r0 + 16; k0 += 8) {
                        uint32_t a[4], b[2];
                        const int ra = r0 + g, rb = r0 + g + 8, ka = k0 + t4, kb2 = k0 + t4 + 4;
                        a[0] = tc::f2tf32(ka <= ra ? MP[ra * LDM + ka] : 0.f);
                        a[1] = tc::f2tf32(ka <= rb ? MP[rb * LDM + ka] : 0.f);
                        a[2] = tc::f2tf32(kb2 <= ra ? MP[ra * LDM + kb2] : 0.f);
                        a[3] = tc::f2tf32(kb2 <= rb ? MP[rb * LDM + kb2] : 0.f);
                        b[0] = tc::f2tf32(E[ka * LDX + n0 + g]);
                        b[1] = tc::f2tf32(E[kb2 * LDX + n0 + g]);
                        tc::mma_tf32(c, a, b);
                    }
                }
                each16x8(r0, n0, c, [&](int t, int j, float v) {
                    if (t < n) ko[(size_t)(c0 + t) * DD + j] = __float2bfloat16_rn(v);
                });
            }
        }
        if (tid < C) vw[tid] = __expf(GC - vG[tid]) * veta[tid];
        __syncthreads();
        // ---- S_end = e^{G_C} S0 + E^T D_w X (d x d, K = C)
        {
            constexpr int NST = (DD / 16) * (DD / 8), PER = NST / (NTHS / 32);  // 16 x 8 tiles, per warp
            float c[PER][4];
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int tt = warp * PER + q, r0 = (tt / (DD / 8)) * 16, n0 = (tt % (DD / 8)) * 8;
#pragma unroll
                for (int e = 0; e < 4; ++e) c[q][e] = 0.f;
                // A(j, s) = E[s][j] w_s: scale X's rows by w instead (B(s, i) = w_s X[s][i])
                const int g = lane >> 2, t4 = lane & 3;
                for (int k0 = 0; k0 < C; k0 += 8) {
                    uint32_t a[4], b[2];
                    a[0] = tc::f2tf32(E[(k0 + t4) * LDX + r0 + g]);
                    a[1] = tc::f2tf32(E[(k0 + t4) * LDX + r0 + g + 8]);
                    a[2] = tc::f2tf32(E[(k0 + t4 + 4) * LDX + r0 + g]);
                    a[3] = tc::f2tf32(E[(k0 + t4 + 4) * LDX + r0 + g + 8]);
                    b[0] = tc::f2tf32(vw[k0 + t4] * X[(k0 + t4) * LDX + n0 + g]);
                    b[1] = tc::f2tf32(vw[k0 + t4 + 4] * X[(k0 + t4 + 4) * LDX + n0 + g]);
                    tc::mma_tf32(c[q], a, b);
                }
            }
            __syncthreads();  // every warp has read S0 for O
            const float gc = __expf(GC);
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int tt = warp * PER + q, r0 = (tt / (DD / 8)) * 16, n0 = (tt % (DD / 8)) * 8;
                each16x8(r0, n0, c[q], [&](int j, int i, float v) { S0[j * LDX + i] = gc * S0[j * LDX + i] + v; });
            }
        }
    }
    __syncthreads();
    if (p.final_state)
        for (int e = tid; e < DD * DD; e += NTHS) p.final_state[bh * DD * DD + e] = S0[(e / DD) * LDX + e % DD];
}

bool seq_chunk_covers(const FwdParams &p) {
    if (!(p.variant == F1 || p.variant == F1A) || p.dk != p.dv) return false;
    if (!(p.dk == 32 || p.dk == 64 || p.dk == 128)) return false;
    if (!(p.chunk == 16 || p.chunk == 32 || p.chunk == 64 || p.chunk == 128)) return false;
    return !(p.chunk == 128 && p.dk == 128);  // 338 KB of shared memory
}

namespace {

template <int C, int DD>
int launch_c(const FwdParams &p, cudaStream_t s) {
    constexpr size_t bytes = SeqLayout<C, DD>::bytes;
    static_assert(bytes <= 227 * 1024, "shared memory of one block");
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr[dev]) {
        cudaFuncSetAttribute(seq_chunk_kernel<C, DD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (dev >= 0 && dev < 64) attr[dev] = true;
    }
    seq_chunk_kernel<C, DD><<<(unsigned)(p.B * p.H), NTHS, bytes, s>>>(p);
    return 0;
}

template <int DD>
int launch_d(const FwdParams &p, cudaStream_t s) {
    switch (p.chunk) {
        case 16: return launch_c<16, DD>(p, s);
        case 32: return launch_c<32, DD>(p, s);
        case 64: return launch_c<64, DD>(p, s);
    }
    return 1;
}

}  // namespace

int launch_seq_chunk(const FwdParams &p, cudaStream_t s) {
    if (!seq_chunk_covers(p)) return 1;
    if (p.chunk == 128) return p.dk == 32 ? launch_c<128, 32>(p, s) : launch_c<128, 64>(p, s);
    switch (p.dk) {
        case 32: return launch_d<32>(p, s);
        case 64: return launch_d<64>(p, s);
        case 128: return launch_d<128>(p, s);
    }
    return 1;
}

}  // namespace falcon
