// k_chunk_split.cu -- chunk-parallel forward on the tcgen05 tensor cores in
// two kernels (Falcon-1 and Falcon-1A, bf16 inputs, d_k = d_v = 64, chunk 64).
//
// Method: "chunk-parallel: parallel inside chunks, recurrent across chunks"
// (page "Fast Weight Attention：用于持续学习的快速权重注意力", 核心方法 3); only a
// fixed-size state passes between chunks (page "借鉴40年前的设想！…", 02 (2)).
//
// Transition form.  Inside a chunk entered with state S (d_v x d_k), with
// g_t = prod_{r<=t} alpha_r (chunk-local), D_a = diag(g_{t-1}), D_g =
// diag(g_t), causal weights Dm[t,s] = (g_t/g_s) eta_s (s <= t), w_s =
// (g_C/g_s) eta_s, A = X X^T and P = Q X^T:
//   T    = (I + M)^{-1},  M[t,s] = (g_{t-1}/g_s) eta_s A[t,s]   (s < t)
//   W    = T D_a X,  U0 = T Y        (inner-product family: W = 0, U0 = Y)
//   Qt   = D_g Q - (P o Dm) W,  O0 = (P o Dm) U0
//   Phi' = W^T D_w X,  B = U0^T D_w X
// and then, exactly,
//   O = Qt S^T + O0,   S_end = g_C S - S Phi' + B.
// Everything but the last line is independent of S, so it is computed for
// every chunk of every head at once by chunk_local_kernel (one block per
// (head, chunk), two blocks per SM); chunk_chain_kernel (one block per head)
// then walks the chunks with one tensor-core product per chunk on its
// critical path.  Every decay factor is a difference of cumulative logs,
// hence <= 1.
//
// The local kernel leaves, per chunk, a 32 KB image in a stream-ordered
// workspace: [-Phi'^T | Qt] as the 128-byte-swizzled K-major operand tiles
// the tensor core reads (bf16), then O0^T and B (bf16, [col/8][row][8], so
// that thread j of the chain kernel reads its row with conflict-free 16-byte
// loads), and g_C in a separate float array.  The chain kernel copies the
// images back with untiled bulk copies into 1024-byte aligned shared memory,
// where the swizzle pattern is the one the local kernel wrote.
//
// Every tcgen05 operand is K-major (rows of 128 bytes, 128-byte swizzle), so
// each product is laid out as D = A B^T with both operands stored row-wise;
// the transposed operands are made by the tensor core itself (A = [.; I]):
//   G1  A=[X;Q]           B=X            -> A (lanes 0-63), P (lanes 64-127)
//   GT  A=[I;.] B=Y -> Y^T (lanes 0-63);  A=[.;I] B=X -> X^T (lanes 64-127)
//       CUDA cores: M, P o Dm, T = (I+M)^{-1} (16x16 blocked inversion, fp32)
//   G2  A=[Y^T;(D_a X)^T] B=T            -> U0^T (lanes 0-63), W^T (64-127)
//   G3  A=[P o Dm;(D_w X)^T] B=W^T       -> (P o Dm)W (0-63), Phi'^T (64-127)
//   G4  A=[U0^T;W^T]      B=[P o Dm;(D_w X)^T] -> [O0^T | B] (lanes 0-63),
//       issued with G3 (neither reads the other's result)
// and in the chain kernel
//   G5  A=[S;S]           B=[-Phi'^T;Qt] -> [-S Phi' | O^T - O0^T], both
//       lane halves (the state warps read lanes 0-63, the output warps 64-127).
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

constexpr int CH = 64;  // chunk
constexpr int DD = 64;  // d_k = d_v
constexpr uint32_t TILE = 8192;     // 64 rows x 128 bytes
constexpr uint32_t IMG = 4 * TILE;  // per-chunk workspace image
constexpr uint64_t kWaitNs = 2000000000ull;  // bounded waits: two seconds

// ------------------------------------------------------------ local kernel
constexpr int NTH1 = 256;
constexpr int ISSUER1 = 128;  // issues every MMA of the local kernel (warp 4)
constexpr uint32_t LDF = 68;  // fp32 row stride of M / T (conflict-free float4 rows and m16n8k8 fragments)
constexpr uint32_t LDZ = 36;
// shared memory (bytes from a 1024-aligned base).  Two sets of input tiles
// (the unit being computed and the next one, prefetched); the three tiles of
// a set are also the staging area of its output image, in image order:
//   X  raw keys -> X in place; inverse scratch; then -Phi'^T
//   Q  Q; then Qt in place
//   V  raw values Y; then bf16 T; then O0^T
constexpr uint32_t L_SET = 3 * TILE;  // set k at k * L_SET: X, Q, V
constexpr uint32_t L_XT = 6 * TILE;   // [Y^T ; (D_a X)^T]
constexpr uint32_t L_A3 = 8 * TILE;   // [P o Dm ; (D_w X)^T]
constexpr uint32_t L_MF = 10 * TILE;  // fp32 M, inverted in place to T; then [U0^T ; W^T]; then B
constexpr uint32_t L_VEC = L_MF + 64 * LDF * 4;  // per-token vectors and scalars
constexpr uint32_t L_BAR = L_VEC + 11 * 64 * 4;
constexpr uint32_t L_SMEM = L_BAR + 64 + 1024;  // + alignment slack
static_assert(2 * TILE <= 64 * LDF * 4, "[U0^T;W^T] must fit over fp32 T");
static_assert(32 * LDZ * 4 <= TILE, "inverse scratch must fit over the samples");
// tensor-memory columns (128 allocated; reused once consumed)
constexpr uint32_t TMEM1 = 256;  // two blocks per SM hold all 512 columns
// G3 and G4 do not depend on each other: the regression family issues both
// after G2 (columns 0-63 and 128-255), under one commit
constexpr uint32_t C_G1 = 0, C_G2 = 64, C_G3 = 0, C_G4 = 128;
// factorised decays e^{G_a - G_b} = e^{G_a - G_ref} e^{G_ref - G_b} need every
// factor inside the fp32 range: used while the chunk's log-decay G_C > -80
constexpr float kFactorMinLogDecay = -80.f;

// ------------------------------------------------------------ chain kernel
constexpr int NTH2 = 320;  // warps 0-7 compute, warp 8 copies, warp 9 issues the products
constexpr int NST = 4;     // image stages in flight
constexpr int NSA = 3;     // bf16 [S ; S] operand buffers (chunk index mod 3), 16 KB each
constexpr uint32_t S_SA = NST * IMG;
constexpr uint32_t S_GC = S_SA + NSA * 2 * TILE;  // g_C per stage
constexpr uint32_t S_BAR = S_GC + 64;
constexpr uint32_t S_SMEM = S_BAR + 256 + 1024;
// chain tensor memory: two accumulators of 128 columns (chunk parity), each
// [-S Phi' | O^T - O0^T] (the inner-product family uses the second half only)

__device__ unsigned int g_split_wait_timeouts;

#ifdef FALCON_TC_DEBUG
__device__ long long *g_split_tim;
// local kernel: per-phase clocks of three blocks, start/end time of every block
#define LDBG_INIT()                                                                        \
    long long *const dbg_tim_ = g_split_tim;                                               \
    const int dbg_w_ = blockIdx.x == 0 ? 0 : blockIdx.x == 1500 ? 1 : blockIdx.x == 3071 ? 2 : -1
#define LTIM(k)                                                                            \
    do {                                                                                   \
        if (dbg_tim_ && dbg_w_ >= 0 && threadIdx.x == 0) dbg_tim_[dbg_w_ * 32 + (k)] = clock64(); \
    } while (0)
// the same by thread t_ (the product windows: issued by ISSUER1, seen by thread 64)
#define LTIMX(t_, k)                                                                         \
    do {                                                                                     \
        if (dbg_tim_ && dbg_w_ >= 0 && threadIdx.x == (t_)) dbg_tim_[dbg_w_ * 32 + (k)] = clock64(); \
    } while (0)
#define LBLK(k)                                                                      \
    do {                                                                             \
        if (dbg_tim_ && threadIdx.x == 0 && blockIdx.x < 4096) {                     \
            unsigned smid_;                                                          \
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid_));                       \
            dbg_tim_[1024 + blockIdx.x * 4 + (k)] = (long long)tc::globaltimer_ns(); \
            dbg_tim_[1024 + blockIdx.x * 4 + 2] = smid_;                             \
        }                                                                            \
    } while (0)
// chain kernel: block 0, chunk c < 32, event k < 8
#define CDBG_INIT() long long *const dbg_ctim_ = blockIdx.x == 0 ? g_split_tim : nullptr
#define CTIM(c, k)                                                                  \
    do {                                                                            \
        if (dbg_ctim_ && (c) < 32) dbg_ctim_[128 + (c) * 16 + (k)] = clock64();     \
    } while (0)
#else
#define LDBG_INIT()
#define CDBG_INIT()
#define LTIM(k)
#define LTIMX(t_, k)
#define LBLK(k)
#define CTIM(c, k)
#endif

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

// Tensor maps of q, k, v: 3-D [B*H][L][64] bf16, boxes of 64 x 64, 128-byte swizzle.
struct SplitMaps {
    CUtensorMap q, k, v;
};

// D = A B^T over K = 64 (four K=16 slices), both operands K-major and
// 128-byte swizzled; M = 128, N = 64 or 128.  Each descriptor is built once
// and advanced per slice.
__device__ __forceinline__ void issue_gemm(uint32_t d_tmem, uint32_t a_saddr, uint32_t b_saddr, int N,
                                           bool accumulate) {
    tc::mma_k64(d_tmem, tc::sdesc_sw128(a_saddr, 16, 1024), tc::sdesc_sw128(b_saddr, 16, 1024),
                tc::idesc_bf16(128, N, 0, 0), accumulate);
}

// One warp: C (16 x 8) = A (16 x K, rows of stride lda) * B (K x 8, rows of
// stride ldb), K a multiple of 8, fp32 in shared memory, TF32 products.
template <int K>
__device__ __forceinline__ void warp_gemm_16x8(const float *A, int lda, const float *B, int ldb, float (&c)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    c[0] = c[1] = c[2] = c[3] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t a[4], b[2];
        a[0] = tc::f2tf32(A[g * lda + k0 + t]);
        a[1] = tc::f2tf32(A[(g + 8) * lda + k0 + t]);
        a[2] = tc::f2tf32(A[g * lda + k0 + t + 4]);
        a[3] = tc::f2tf32(A[(g + 8) * lda + k0 + t + 4]);
        b[0] = tc::f2tf32(B[(k0 + t) * ldb + g]);
        b[1] = tc::f2tf32(B[(k0 + t + 4) * ldb + g]);
        tc::mma_tf32(c, a, b);
    }
}

// Write a 16 x 8 accumulator fragment (times `scale`) to C (row stride ldc).
__device__ __forceinline__ void warp_store_16x8(float *C, int ldc, const float (&c)[4], float scale) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    C[g * ldc + 2 * t] = scale * c[0];
    C[g * ldc + 2 * t + 1] = scale * c[1];
    C[(g + 8) * ldc + 2 * t] = scale * c[2];
    C[(g + 8) * ldc + 2 * t + 1] = scale * c[3];
}

// Byte offset of the 16-byte group (row r, columns 8*g8 .. 8*g8+7) in the
// [col/8][row][8] bf16 layout of O0^T and B.
__device__ __forceinline__ uint32_t rowmajor8(int r, int g8) { return (uint32_t)((g8 * 64 + r) * 16); }

}  // namespace

// ============================================================ local kernel
namespace {

// Transposed copy of four 8x8 blocks of a 64x64 bf16 tile (128-byte rows,
// 128-byte swizzle): source row block rb, 16-byte chunks cb0..cb0+3 ->
// destination row blocks cb0..cb0+3, chunk rb.  Each element is scaled by
// scale[source row] on the way (rounded once to bf16); scale == nullptr
// copies.  Whole warp.
__device__ __forceinline__ void transpose4(uint32_t src, int rb, int cb0, uint32_t dst, const float *scale,
                                           uint32_t dst2, const float *scale2) {
    const int lane = threadIdx.x & 31, m = lane >> 3, i = lane & 7;
    uint32_t r[4];
    tc::ldsm_x4_trans(src + (uint32_t)(rb * 8 + i) * 128u + ((uint32_t)((cb0 + m) ^ i) << 4), r);
    const uint32_t dofs = (uint32_t)((cb0 + m) * 8 + i) * 128u + ((uint32_t)(rb ^ i) << 4);
    const int sr = rb * 8 + 2 * (lane & 3);  // source rows of this thread's pairs
    if (scale == nullptr) {
        tc::stsm_x4(dst + dofs, r);
    } else {
        const float s0 = scale[sr], s1 = scale[sr + 1];
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r[k]));
            const __nv_bfloat162 h = __floats2bfloat162_rn(f.x * s0, f.y * s1);
            o[k] = *reinterpret_cast<const uint32_t *>(&h);
        }
        tc::stsm_x4(dst + dofs, o);
    }
    if (dst2) {
        const float s0 = scale2[sr], s1 = scale2[sr + 1];
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r[k]));
            const __nv_bfloat162 h = __floats2bfloat162_rn(f.x * s0, f.y * s1);
            o[k] = *reinterpret_cast<const uint32_t *>(&h);
        }
        tc::stsm_x4(dst2 + dofs, o);
    }
}

}  // namespace

// Persistent: block i computes units i, i + gridDim.x, ... (unit = bh *
// nchunks + c), the inputs of its next unit loading while it computes one.
__global__ void __launch_bounds__(NTH1, 2)
    chunk_local_kernel(FwdParams p, const __grid_constant__ SplitMaps maps, uint8_t *img_ws, float *gc_ws) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *Mf = reinterpret_cast<float *>(sm + L_MF);  // M, then T in place
    float *vec = reinterpret_cast<float *>(sm + L_VEC);
    float *v_la = vec, *v_eta = vec + 64, *v_G = vec + 128, *v_gm1 = vec + 192, *v_gt = vec + 256,
          *v_w = vec + 320, *v_lsc = vec + 384, *v_a = vec + 448, *v_b = vec + 512, *v_c = vec + 576,
          *v_sc = vec + 640;  // v_sc[1]: factorised-decay flag; v_sc[8..15]: per-warp log-decay sums
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L_BAR);        // MMA completion
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L_BAR + 8);
    uint64_t *tbar = reinterpret_cast<uint64_t *>(sm + L_BAR + 16);  // [2] TMA arrival per input set

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, chalf = warp >> 2;
    const int row = quarter * 32 + lane;  // accumulator row (tensor-memory lane) of this thread
    const bool reg = p.variant == F1;
    const int L = p.L;
    const int nch = (L + CH - 1) / CH;
    const int units = p.B * p.H * nch;
    LDBG_INIT();
    LBLK(0);
    LTIM(0);

    // loads of unit u into input set k: raw keys (row t <- key c0+t-1 under
    // the prefix pair, key c0+t under the same-step pair; the key before the
    // sequence start and rows past its end read as zeros), q, v
    auto load_unit = [&](int u, int k) {
        const int ubh = u / nch, uc0 = (u - ubh * nch) * CH;
        const uint32_t o = sbase + (uint32_t)k * L_SET;
        tc::mbar_arrive_expect_tx(&tbar[k], 3 * TILE);
        tc::tma_load_3d(o, &maps.k, 0, p.pairing == 0 ? uc0 - 1 : uc0, ubh, &tbar[k]);
        tc::tma_load_3d(o + TILE, &maps.q, 0, uc0, ubh, &tbar[k]);
        tc::tma_load_3d(o + 2 * TILE, &maps.v, 0, uc0, ubh, &tbar[k]);
    };
    // beta and lambda of a unit travel in registers, loaded a unit ahead
    auto load_scalars = [&](int u, __nv_bfloat16 &braw, float &lraw) {
        braw = __float2bfloat16_rn(0.f);
        lraw = 0.f;
        if (u >= units) return;
        const int ubh = u / nch, uc0 = (u - ubh * nch) * CH;
        // token t = tid / 4 on the first of the four threads of sample row t
        if ((tid & 3) == 0) {
            if (uc0 + (tid >> 2) < L) braw = static_cast<const __nv_bfloat16 *>(p.beta)[(size_t)ubh * L + uc0 + (tid >> 2)];
            lraw = p.lambda[ubh % p.H];
        }
    };

    int loads0 = 0, loads1 = 0;  // loads issued into each input set (thread 0)
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(&tbar[0], 1);
        tc::mbar_init(&tbar[1], 1);
        tc::fence_mbar_init();
        if ((int)blockIdx.x < units) {
            load_unit(blockIdx.x, 0);
            loads0 = 1;
        }
    }
    __syncwarp();
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TMEM1);
        tc::tmem_relinquish();
    }
    __nv_bfloat16 beta_raw;
    float lam_raw;
    load_scalars(blockIdx.x, beta_raw, lam_raw);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(quarter * 32) << 16);  // this warp's lanes
    LTIM(1);

    bool ok = true;
    uint32_t phase = 0;  // MMA-completion parity
    int n = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++n) {
    const int set = n & 1;
    const uint32_t oX = (uint32_t)set * L_SET, oQ = oX + TILE, oV = oX + 2 * TILE;
    float *Zf = reinterpret_cast<float *>(sm + oX);  // inverse scratch over the consumed samples
    const int un = u + gridDim.x;
    if (tid == 0) {
        // the previous image (the other set's tiles and B over M) has been
        // read out of shared memory: both may be written again
        tc::bulk_wait_read();
        if (un < units) {
            load_unit(un, set ^ 1);
            if (set) ++loads0; else ++loads1;
        }
    }
    __nv_bfloat16 beta_next;
    float lam_next;
    load_scalars(un, beta_next, lam_next);

    ok = tc::mbar_wait_timeout(&tbar[set], (n >> 1) & 1, kWaitNs);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    LTIM(2);
    {
        // ---- samples x_t = phi(k_{t-1}) in place (four threads per row t), the
        //      steps and log decays of the rows, and their cumulative sums
        //      inside each warp (eight rows per warp)
        {
            const int r = tid >> 2, part = tid & 3;
            // x of a continued segment's first token is the carried phi(k), as given
            const bool carried = r == 0 && p.x_prev != nullptr && u % nch == 0;
            float xr[16];
            float ss = 0.f;
#pragma unroll
            for (int c16 = 0; c16 < 2; ++c16) {
                if (carried) {
                    const float *xp = p.x_prev + (size_t)(u / nch) * DD + part * 16 + c16 * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) xr[c16 * 8 + e] = xp[e];
                } else {
                    unpack8(*reinterpret_cast<const uint4 *>(sm + oX + tc::sw128(r, part * 2 + c16)), &xr[c16 * 8]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) ss += xr[c16 * 8 + e] * xr[c16 * 8 + e];
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            const float inv = (carried || p.phi != 0) ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
            const float sq = ss * inv * inv;  // |x_t|^2: 1 up to rounding, 0 for an empty sample
#pragma unroll
            for (int e = 0; e < 16; ++e) xr[e] *= inv;
#pragma unroll
            for (int c16 = 0; c16 < 2; ++c16)
                *reinterpret_cast<uint4 *>(sm + oX + tc::sw128(r, part * 2 + c16)) = pack8(&xr[c16 * 8]);
            // eta = beta / (eps + n) (0 for an empty sample), alpha = max(1 - eta lambda, 2^-20)
            const float beta_r = __shfl_sync(0xffffffffu, __bfloat162float(beta_raw), lane & ~3);
            const float lam = __shfl_sync(0xffffffffu, lam_raw, lane & ~3);
            const float eta = sq > 0.f ? __fdividef(beta_r, p.eps + sq) : 0.f;
            const float la = __logf(fmaxf(1.f - eta * lam, kAlphaFloor));
            float run = la;  // inclusive sum over this warp's rows (lanes 4k hold row 8w+k)
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run += y;
            }
            if (part == 0) {
                v_la[r] = la;
                v_lsc[r] = run;
                v_eta[r] = eta;
            }
            if (lane == 28) v_sc[8 + warp] = run;
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        LTIM(3);
        // ---- G1 [X;Q] X^T -> A (lanes 0-63), P (lanes 64-127), while the decays are formed
        if (tid == ISSUER1) {
            tc::fence_after_sync();
            LTIMX(ISSUER1, 24);
            issue_gemm(tbase + C_G1, sbase + oX, sbase + oX, 64, false);
            tc::mma_commit(bar);
        }
        __syncwarp();
        if (tid < 64) {
            // ---- token t: cumulative log decay G_t and the decay vectors
            const int t = tid;
            const float4 wa = *reinterpret_cast<const float4 *>(v_sc + 8);
            const float4 wb = *reinterpret_cast<const float4 *>(v_sc + 12);
            const float wt[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            float off = 0.f, GC = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                if (w < (t >> 3)) off += wt[w];
                GC += wt[w];
            }
            const float Gr = v_lsc[31] + (wt[0] + wt[1] + wt[2]);  // G_31, the factorisation's reference
            const float Gt = v_lsc[t] + off, Gm = Gt - v_la[t];    // G_t, G_{t-1}
            const float eta = v_eta[t];
            v_G[t] = Gt;
            v_gm1[t] = __expf(Gm);
            v_gt[t] = __expf(Gt);
            v_w[t] = __expf(GC - Gt) * eta;
            // e^{G_{t-1} - G_s} = a_t b_s / eta_s and e^{G_t - G_s} = c_t b_s / eta_s
            v_a[t] = __expf(Gm - Gr);
            v_c[t] = __expf(Gt - Gr);
            v_b[t] = eta * __expf(Gr - Gt);
            if (t == 0) {
                gc_ws[u] = __expf(GC);
                v_sc[1] = GC > kFactorMinLogDecay ? 1.f : 0.f;
            }
        } else if (warp >= 4) {
            // ---- Y^T -> XT rows 0-63 (warps 4-7, two source row blocks each)
            const int rb = 2 * (warp - 4);
            transpose4(sbase + oV, rb, 0, sbase + L_XT, nullptr, 0, nullptr);
            transpose4(sbase + oV, rb, 4, sbase + L_XT, nullptr, 0, nullptr);
            transpose4(sbase + oV, rb + 1, 0, sbase + L_XT, nullptr, 0, nullptr);
            transpose4(sbase + oV, rb + 1, 4, sbase + L_XT, nullptr, 0, nullptr);
        }
        LTIM(16);
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        LTIMX(64, 28);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        LTIM(4);
    }
    if (ok) {
        tc::fence_after_sync();
        // ---- (D_w X)^T -> A3 rows 64-127 and (D_a X)^T -> XT rows 64-127
        //      (regression), source row block = warp
        transpose4(sbase + oX, warp, 0, sbase + L_A3 + TILE, v_w, reg ? sbase + L_XT + TILE : 0, v_gm1);
        transpose4(sbase + oX, warp, 4, sbase + L_A3 + TILE, v_w, reg ? sbase + L_XT + TILE : 0, v_gm1);
        LTIM(5);
        // rows 0-63: M[t][s] = (g_{t-1}/g_s) eta_s A[t][s] for s < t (fp32, regression only);
        // rows 64-127: (P o Dm)[t][s] = (g_t/g_s) eta_s P[t][s] for s <= t (bf16).
        const bool mrow = quarter < 2;
        const int t = mrow ? row : row - 64;
        const bool fact = v_sc[1] != 0.f;
        if (!mrow || reg) {
            const float rowf = mrow ? v_a[t] : v_c[t];
            const float gref = mrow ? (t > 0 ? v_G[t - 1] : 0.f) : v_G[t];
            const int tlim = mrow ? t : t + 1;  // s < tlim
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16], m[16];
                tc::tmem_ld16(tlane + C_G1 + cs * 16, v);
                if (fact) {
                    float bs[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 b4 = reinterpret_cast<const float4 *>(v_b)[cs * 4 + q];
                        bs[q * 4 + 0] = b4.x; bs[q * 4 + 1] = b4.y; bs[q * 4 + 2] = b4.z; bs[q * 4 + 3] = b4.w;
                    }
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) m[i] = cs * 16 + i < tlim ? rowf * (bs[i] * v[i]) : 0.f;
                } else {
                    // every factor as one exponential of a difference, argument clamped to <= 0
                    float gs[16], es[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 g = reinterpret_cast<const float4 *>(v_G)[cs * 4 + q];
                        const float4 e = reinterpret_cast<const float4 *>(v_eta)[cs * 4 + q];
                        gs[q * 4 + 0] = g.x; gs[q * 4 + 1] = g.y; gs[q * 4 + 2] = g.z; gs[q * 4 + 3] = g.w;
                        es[q * 4 + 0] = e.x; es[q * 4 + 1] = e.y; es[q * 4 + 2] = e.z; es[q * 4 + 3] = e.w;
                    }
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float x = __expf(fminf(gref - gs[i], 0.f)) * es[i] * v[i];
                        m[i] = cs * 16 + i < tlim ? x : 0.f;
                    }
                }
                if (mrow) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4 *>(Mf + t * LDF + cs * 16 + q * 4) =
                            make_float4(m[q * 4], m[q * 4 + 1], m[q * 4 + 2], m[q * 4 + 3]);
                } else {
                    *reinterpret_cast<uint4 *>(sm + L_A3 + tc::sw128(t, cs * 2)) = pack8(&m[0]);
                    *reinterpret_cast<uint4 *>(sm + L_A3 + tc::sw128(t, cs * 2 + 1)) = pack8(&m[8]);
                }
            }
        } else {
            // inner-product family, rows 0-63: no M; Qt = D_g Q in place (G1 has read Q)
            const float g = v_gt[t];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float q8[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + oQ + tc::sw128(t, chalf * 4 + cc)), q8);
#pragma unroll
                for (int i = 0; i < 8; ++i) q8[i] *= g;
                *reinterpret_cast<uint4 *>(sm + oQ + tc::sw128(t, chalf * 4 + cc)) = pack8(q8);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        LTIM(6);
    }

    uint32_t a4 = sbase + L_XT;  // A of G4: [U0^T; W^T], or [Y^T; .] for the A family
    if (ok && reg) {
        // ---- T = (I + M)^{-1} in place over M.  Diagonal 16x16 blocks by
        //      forward substitution (warp b, lane = column); the off-diagonal
        //      blocks by T_ij = -T_ii (M_i. T_.j) with TF32 warp MMAs.  M's
        //      upper triangle holds zeros, which T's upper triangle keeps.
        if (warp < 4 && lane < 16) {
            const int b0 = warp * 16, j = lane;
            float tcol[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                // row i of the diagonal block, four float4 loads (broadcast across the lanes)
                float mr[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 m4 = *reinterpret_cast<const float4 *>(Mf + (b0 + i) * LDF + b0 + q * 4);
                    mr[q * 4] = m4.x; mr[q * 4 + 1] = m4.y; mr[q * 4 + 2] = m4.z; mr[q * 4 + 3] = m4.w;
                }
                float acc[4] = {(i == j) ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s = 0; s < i; ++s) acc[s & 3] -= mr[s] * tcol[s];
                tcol[i] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            }
            __syncwarp(0x0000ffffu);  // every lane has read the block before any writes it
#pragma unroll
            for (int i = 0; i < 16; ++i) Mf[(b0 + i) * LDF + b0 + j] = tcol[i];
        }
        __syncthreads();
        LTIM(20);
        if (warp < 4) {  // blocks (1,0) [warps 0,1] and (3,2) [warps 2,3]; warp = 8 columns
            const int pb = warp >> 1, nt = warp & 1;
            const int r0 = pb ? 48 : 16, q0 = pb ? 32 : 0;
            float *zw = Zf + warp * 16 * 8;  // this warp's 16 x 8 scratch
            float c4[4];
            warp_gemm_16x8<16>(Mf + r0 * LDF + q0, LDF, Mf + q0 * LDF + q0 + nt * 8, LDF, c4);
            warp_store_16x8(zw, 8, c4, 1.f);
            tc::named_sync(2, 128);  // both warps of a block have read M_ij before it is overwritten
            warp_gemm_16x8<16>(Mf + r0 * LDF + r0, LDF, zw, 8, c4);
            warp_store_16x8(Mf + r0 * LDF + q0 + nt * 8, LDF, c4, -1.f);
        }
        __syncthreads();
        LTIM(21);
        // 32x32 block (rows 32-63, cols 0-31); warp = one 16x8 tile
        const int rb = warp >> 2, cb = (warp >> 1) & 1, nt = warp & 1;
        {   // Z = M_HL T_LL
            float c4[4];
            warp_gemm_16x8<32>(Mf + (32 + rb * 16) * LDF, LDF, Mf + cb * 16 + nt * 8, LDF, c4);
            warp_store_16x8(Zf + rb * 16 * LDZ + cb * 16 + nt * 8, LDZ, c4, 1.f);
        }
        __syncthreads();
        LTIM(22);
        {   // T_HL = -T_HH Z, straight to its bf16 tile (rows 32-63, columns 0-31 of T)
            float c4[4];
            warp_gemm_16x8<32>(Mf + (32 + rb * 16) * LDF + 32, LDF, Zf + cb * 16 + nt * 8, LDZ, c4);
            const int g = lane >> 2, t4 = lane & 3, r0 = 32 + rb * 16 + g, ch = cb * 2 + nt;
            const __nv_bfloat162 lo = __floats2bfloat162_rn(-c4[0], -c4[1]), hi = __floats2bfloat162_rn(-c4[2], -c4[3]);
            *reinterpret_cast<__nv_bfloat162 *>(sm + oV + tc::sw128(r0, ch) + t4 * 4) = lo;
            *reinterpret_cast<__nv_bfloat162 *>(sm + oV + tc::sw128(r0 + 8, ch) + t4 * 4) = hi;
        }
        LTIM(23);
        {   // the rest of T to bf16 over the consumed values: thread = (row, 16 columns)
            const int r = tid >> 2, part = tid & 3;
#pragma unroll
            for (int c16 = 0; c16 < 2; ++c16) {
                if (r >= 32 && part < 2) break;  // T_HL, written above
                float t8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = part * 16 + c16 * 8 + e;
                    t8[e] = s <= r ? Mf[r * LDF + s] : 0.f;
                }
                *reinterpret_cast<uint4 *>(sm + oV + tc::sw128(r, part * 2 + c16)) = pack8(t8);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        LTIM(7);

        // ---- G2: [Y^T;(D_a X)^T] T^T -> U0^T (lanes 0-63), W^T (lanes 64-127)
        if (tid == ISSUER1) {
            tc::fence_after_sync();
            LTIMX(ISSUER1, 25);
            issue_gemm(tbase + C_G2, sbase + L_XT, sbase + oV, 64, false);
            tc::mma_commit(bar);
        }
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        LTIMX(64, 29);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        if (ok) {
            tc::fence_after_sync();
            // [U0^T ; W^T] over the consumed fp32 T
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16];
                tc::tmem_ld16(tlane + C_G2 + cs * 16, v);
                tc::tmem_wait_ld();
                *reinterpret_cast<uint4 *>(sm + L_MF + tc::sw128(row, cs * 2)) = pack8(&v[0]);
                *reinterpret_cast<uint4 *>(sm + L_MF + tc::sw128(row, cs * 2 + 1)) = pack8(&v[8]);
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            LTIM(8);

            // ---- G3: [P o Dm;(D_w X)^T] W -> (P o Dm) W (lanes 0-63), Phi'^T (lanes 64-127)
            //      G4: [U0^T;W^T] [P o Dm;(D_w X)^T]^T -> [O0^T | B] (lanes 0-63), at once
            if (tid == ISSUER1) {
                tc::fence_after_sync();
                LTIMX(ISSUER1, 26);
                issue_gemm(tbase + C_G3, sbase + L_A3, sbase + L_MF + TILE, 64, false);
                issue_gemm(tbase + C_G4, sbase + L_MF, sbase + L_A3, 128, false);
                tc::mma_commit(bar);
            }
            ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
            LTIMX(64, 30);
            phase ^= 1;
            ok = __syncthreads_and(ok);
            LTIM(9);
        }
        if (ok) {
            tc::fence_after_sync();
            const bool qrow = quarter < 2;
            const float g = qrow ? v_gt[row] : -1.f;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16];
                tc::tmem_ld16(tlane + C_G3 + cs * 16, v);
                tc::tmem_wait_ld();
                if (qrow) {  // Qt = D_g Q - (P o Dm) W, in place over Q
                    float q8[8];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        unpack8(*reinterpret_cast<const uint4 *>(sm + oQ + tc::sw128(row, cs * 2 + hh)), q8);
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[hh * 8 + i] = g * q8[i] - v[hh * 8 + i];
                    }
                    *reinterpret_cast<uint4 *>(sm + oQ + tc::sw128(row, cs * 2)) = pack8(&v[0]);
                    *reinterpret_cast<uint4 *>(sm + oQ + tc::sw128(row, cs * 2 + 1)) = pack8(&v[8]);
                } else {  // -Phi'^T over the consumed samples
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = -v[i];
                    *reinterpret_cast<uint4 *>(sm + oX + tc::sw128(row - 64, cs * 2)) = pack8(&v[0]);
                    *reinterpret_cast<uint4 *>(sm + oX + tc::sw128(row - 64, cs * 2 + 1)) = pack8(&v[8]);
                }
            }
        }
        a4 = sbase + L_MF;
    }
    if (reg) {  // (the inner-product family's G4 operands were complete at the last barrier)
        tc::fence_proxy_async();
        tc::fence_before_sync();
        ok = __syncthreads_and(ok);
    }
    LTIM(10);

    if (ok && !reg) {  // (the regression family issued G4 with G3)
        // ---- G4: [Y^T; .] [P o Dm; (D_w X)^T]^T -> [O0^T | B] (lanes 0-63)
        if (tid == ISSUER1) {
            tc::fence_after_sync();
            LTIMX(ISSUER1, 27);
            issue_gemm(tbase + C_G4, a4, sbase + L_A3, 128, false);
            tc::mma_commit(bar);
        }
        ok = tc::mbar_wait_timeout(bar, phase, kWaitNs);
        LTIMX(64, 31);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        LTIM(11);
    }
    if (ok) {
        tc::fence_after_sync();
        if (quarter < 2) {  // O0^T -> over T (bf16), B -> over [U0^T;W^T]; both [col/8][row][8]
            const int j = row;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t dst = part ? L_MF : oV;
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    const int cs = chalf * 2 + k2;
                    float v[16];
                    tc::tmem_ld16(tlane + C_G4 + part * 64 + cs * 16, v);
                    tc::tmem_wait_ld();
                    *reinterpret_cast<uint4 *>(sm + dst + rowmajor8(j, cs * 2)) = pack8(&v[0]);
                    *reinterpret_cast<uint4 *>(sm + dst + rowmajor8(j, cs * 2 + 1)) = pack8(&v[8]);
                }
            }
        }
        tc::fence_proxy_async();  // staged image -> the bulk-copy engine
        __syncthreads();
        LTIM(12);
        if (tid == 0) {
            uint8_t *dst = img_ws + (size_t)u * IMG;
            if (reg)
                tc::bulk_store(dst, sbase + oX, 3 * TILE);  // -Phi'^T | Qt | O0^T
            else  // no -Phi'^T for the inner-product family
                tc::bulk_store(dst + TILE, sbase + oQ, 2 * TILE);
            tc::bulk_store(dst + 3 * TILE, sbase + L_MF, TILE);  // B
            tc::bulk_commit();
        }
        LTIM(13);
    }
    if (!ok) break;
    beta_raw = beta_next;
    lam_raw = lam_next;
    }  // units
    // the chain kernel may be scheduled once every block has got this far
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (tid == 0) {
        tc::bulk_wait_read();  // the last images have been read out of shared memory
        if (!ok) {
            atomicAdd(&g_split_wait_timeouts, 1u);
            // loads still in flight must land before the block leaves
            if (loads0 > 0) (void)tc::mbar_wait_timeout(&tbar[0], (loads0 - 1) & 1, kWaitNs);
            if (loads1 > 0) (void)tc::mbar_wait_timeout(&tbar[1], (loads1 - 1) & 1, kWaitNs);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, TMEM1);
    LTIM(14);
    LBLK(1);
}

// ============================================================ chain kernel
// One block per b*H + h.  Warps 0,1,4,5 (tensor-memory lanes 0-63) carry the
// state, fp32 in registers (thread: row j, 32 of its columns); warps 2,3,6,7
// (lanes 64-127) finish the outputs; warp 8 streams the images; warp 9
// issues the products.  S_c sits, as a bf16 [S;S] operand, in buffer c mod 3.
// Regression family: one product per chunk, [S;S] [-Phi'^T;Qt]^T into
// accumulator c & 1, then the state warps form S_{c+1} in fp32, write its
// copy and release the issuer through a named barrier.  Inner-product family:
// no product is on the chain (S_{c+1} = g_C S_c + B_c); the state warps run
// up to three chunks ahead, and each output product Qt_c S_c^T waits for its
// S_c copy (sready) and frees its buffer on completion (sfree).
namespace {

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (*abort_flag) return false;
    if (tc::mbar_wait_timeout(bar, parity, kWaitNs)) return true;
    *abort_flag = 1;
    return false;
}

}  // namespace

__global__ void __launch_bounds__(NTH2, 1)
    chunk_chain_kernel(FwdParams p, const uint8_t *img_ws, const float *gc_ws) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *gcs = reinterpret_cast<float *>(sm + S_GC);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + S_BAR);  // [NST] image landed
    uint64_t *empty = full + NST;                                // [NST] image consumed (8 warps)
    uint64_t *mma_o = empty + NST;                               // [2] the chunk's product done
    uint64_t *accfree = mma_o + 2;                               // [2] outputs read (4 warps)
    uint64_t *sready = accfree + 2;                              // [NSA] S copy written (inner product)
    uint64_t *sfree = sready + NSA;                              // [NSA] S copy read (inner product)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sfree + NSA);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool reg = p.variant == F1 || p.variant == F3;  // a -Phi'^T tile in the image
    const int L = p.L, nch = (L + CH - 1) / CH;
    const int bh = blockIdx.x;
    const uint8_t *imgs = img_ws + (size_t)bh * nch * IMG;
    const float *gcv = gc_ws + (size_t)bh * nch;
    CDBG_INIT();

    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 8);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&mma_o[b], 1);
            tc::mbar_init(&accfree[b], 4);
        }
        for (int b = 0; b < NSA; ++b) {
            tc::mbar_init(&sready[b], 128);
            tc::mbar_init(&sfree[b], 1);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
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
    // launched as a programmatic dependent of the local kernel: the set-up
    // above overlaps its tail; its images are read only after it completed
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 8) {
        // ---- producer: chunk images into NST stages
        if (lane == 0) {
            const uint32_t off = reg ? 0u : TILE;  // the inner-product family has no -Phi'^T
            int issued = 0;
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST;
                if (c >= NST && !wait_or_abort(&empty[s], ((c / NST) - 1) & 1, abort_flag)) break;
                gcs[s] = gcv[c];
                tc::mbar_arrive_expect_tx(&full[s], IMG - off);
                tc::bulk_load(sbase + s * IMG + off, imgs + (size_t)c * IMG + off, IMG - off, &full[s]);
                CTIM(c, 5);
                issued = c + 1;
            }
            // copies still in flight must land before the block leaves
            for (int c = (issued > NST ? issued - NST : 0); c < issued; ++c)
                (void)tc::mbar_wait_timeout(&full[c % NST], (c / NST) & 1, kWaitNs);
        }
    } else if (warp == 9) {
        // ---- issuer
        if (reg) {
            // one product per chunk: [S;S] [-Phi'^T ; Qt]^T -> [-S Phi' | O^T - O0^T]
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST, b = c & 1;
                const uint32_t stage = sbase + s * IMG, sa = sbase + S_SA + (uint32_t)(c % NSA) * 2 * TILE;
                bool go = true;
                if (lane == 0) {
                    go = wait_or_abort(&full[s], (c / NST) & 1, abort_flag);
                    if (go && c >= 2) go = wait_or_abort(&accfree[b], ((c / 2) - 1) & 1, abort_flag);
                }
                __syncwarp();
                tc::named_sync(1, 160);  // S_c is in operand buffer c mod 3
                if (lane == 0) {
                    CTIM(c, 0);
                    tc::fence_after_sync();
                    if (go) issue_gemm(tbase + b * 128, sa, stage, 128, false);
                    tc::mma_commit(&mma_o[b]);
                    CTIM(c, 9);
                }
                __syncwarp();
            }
        } else if (lane == 0) {
            // inner-product family: nothing on the chain is a product; the
            // state warps run ahead and each output product waits for its S_c
            for (int c = 0; c < nch; ++c) {
                const int b = c & 1;
                const uint32_t stage = sbase + (c % NST) * IMG, sa = sbase + S_SA + (uint32_t)(c % NSA) * 2 * TILE;
                bool go = wait_or_abort(&full[c % NST], (c / NST) & 1, abort_flag);
                if (go) go = wait_or_abort(&sready[c % NSA], (c / NSA) & 1, abort_flag);
                if (go && c >= 2) go = wait_or_abort(&accfree[b], ((c / 2) - 1) & 1, abort_flag);
                CTIM(c, 0);
                tc::fence_after_sync();
                if (go) issue_gemm(tbase + b * 128 + 64, sa, stage + TILE, 64, false);
                tc::mma_commit(&mma_o[b]);
                tc::mma_commit(&sfree[c % NSA]);
            }
        }
    } else {
        const int quarter = warp & 3, chalf = warp >> 2;
        const bool state_warp = quarter < 2;
        const int j = (quarter & 1) * 32 + lane;  // state row (value channel)
        const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16);
        __nv_bfloat16 *ko = static_cast<__nv_bfloat16 *>(p.out) + (size_t)bh * L * DD;

        if (state_warp) {
            // S_0: the carried state of a continued segment, else zeros; its
            // bf16 copy goes to both halves of operand buffer 0
            float S[32];
            if (p.init_state) {
                const float *s0 = p.init_state + ((size_t)bh * DD + j) * DD + chalf * 32;
#pragma unroll
                for (int i = 0; i < 32; ++i) S[i] = s0[i];
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) S[i] = 0.f;
            }
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                const uint4 u4 = pack8(&S[g8 * 8]);
                *reinterpret_cast<uint4 *>(sm + S_SA + tc::sw128(j, chalf * 4 + g8)) = u4;
                *reinterpret_cast<uint4 *>(sm + S_SA + TILE + tc::sw128(j, chalf * 4 + g8)) = u4;
            }
            tc::fence_proxy_async();
            if (reg) {
                tc::named_sync(1, 160);  // S_0 is in operand buffer 0
            } else {
                tc::fence_before_sync();
                tc::mbar_arrive(&sready[0]);
            }
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST;
                const uint8_t *st = sm + s * IMG;
                if (p.states_out) {  // the state entering chunk c, for the backward
                    float *so = p.states_out + (((size_t)bh * nch + c) * DD + j) * DD + chalf * 32;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(so + q * 4) =
                            make_float4(S[q * 4], S[q * 4 + 1], S[q * 4 + 2], S[q * 4 + 3]);
                }
                // B row j (this thread's 32 columns) and g_C while the product runs
                (void)wait_or_abort(&full[s], (c / NST) & 1, abort_flag);
                float bv[32];
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8)
                    unpack8(*reinterpret_cast<const uint4 *>(st + 3 * TILE + rowmajor8(j, chalf * 4 + g8)),
                            &bv[g8 * 8]);
                const float g = gcs[s];
                if (reg) {
                    (void)wait_or_abort(&mma_o[c & 1], (c / 2) & 1, abort_flag);
                    if (tid == 0) CTIM(c, 1);
                    tc::fence_after_sync();
                    float ds[32];
                    tc::tmem_ld32(tl + (c & 1) * 128 + chalf * 32, ds);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) S[i] = g * S[i] + ds[i] + bv[i];
                    tc::fence_before_sync();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) S[i] = g * S[i] + bv[i];
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&empty[s]);
                if (c + 1 < nch) {
                    // bf16 copy of S_{c+1} into both halves of operand buffer (c+1) mod 3,
                    // over S_{c-2}: regression - covered by the -S Phi' commit of chunk c;
                    // inner product - once the output product of chunk c-2 has read it
                    if (!reg && c >= 2) (void)wait_or_abort(&sfree[(c + 1) % NSA], ((c - 2) / NSA) & 1, abort_flag);
                    uint8_t *sa = sm + S_SA + ((c + 1) % NSA) * 2 * TILE;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const uint4 u = pack8(&S[g8 * 8]);
                        *reinterpret_cast<uint4 *>(sa + tc::sw128(j, chalf * 4 + g8)) = u;
                        *reinterpret_cast<uint4 *>(sa + TILE + tc::sw128(j, chalf * 4 + g8)) = u;
                    }
                    tc::fence_proxy_async();
                    if (tid == 0) CTIM(c, 2);
                    if (reg) {
                        tc::named_sync(1, 160);
                    } else {
                        tc::fence_before_sync();
                        tc::mbar_arrive(&sready[(c + 1) % NSA]);
                    }
                }
            }
            if (p.final_state && !*(volatile int *)abort_flag) {
                float *fs = p.final_state + ((size_t)bh * DD + j) * DD + chalf * 32;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4 *>(fs + q * 4) =
                        make_float4(S[q * 4], S[q * 4 + 1], S[q * 4 + 2], S[q * 4 + 3]);
            }
        } else {
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST, b = c & 1;
                const uint8_t *st = sm + s * IMG;
                // ---- outputs of chunk c: O^T = (Qt S^T)^T + O0^T -> out[c0 + t][j]
                (void)wait_or_abort(&full[s], (c / NST) & 1, abort_flag);
                float o0[32];
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8)
                    unpack8(*reinterpret_cast<const uint4 *>(st + 2 * TILE + rowmajor8(j, chalf * 4 + g8)),
                            &o0[g8 * 8]);
                (void)wait_or_abort(&mma_o[b], (c / 2) & 1, abort_flag);
                if (tid == 64) CTIM(c, 4);
                tc::fence_after_sync();
                float ov[32];
                tc::tmem_ld32(tl + b * 128 + 64 + chalf * 32, ov);
                tc::tmem_wait_ld();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(&accfree[b]);
                    tc::mbar_arrive(&empty[s]);
                }
                const int c0 = c * CH, nt = min(CH, L - c0);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = chalf * 32 + i;
                    if (t < nt) ko[(size_t)(c0 + t) * DD + j] = __float2bfloat16_rn(ov[i] + o0[i]);
                }
                if (tid == 64) CTIM(c, 6);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && *(volatile int *)abort_flag) atomicAdd(&g_split_wait_timeouts, 1u);
    if (warp == 0) tc::tmem_dealloc(tbase, 256);
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

// [B*H][L][64] bf16 tensor, 64 x 64 boxes, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap *m, const void *base, int BH, int L) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DD, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)DD * 2, (cuuint64_t)L * DD * 2};
    const cuuint32_t box[3] = {DD, CH, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Multiprocessor count of the current device (the persistent grid's size).
int sm_count() {
    static int counts[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

bool split_chunk_covers(const FwdParams &p) {
    if (!((p.variant == F1 || p.variant == F1A) && p.dk == DD && p.dv == DD && p.chunk == CH)) return false;
    return (size_t)p.B * p.H * ((p.L + CH - 1) / CH) <= 0x7fffffffu;
}

size_t split_chunk_ws_bytes(const FwdParams &p) {
    const size_t units = (size_t)p.B * p.H * ((p.L + CH - 1) / CH);
    return units * IMG + units * sizeof(float);
}

size_t split_chunk_images_ws_bytes(const FwdParams &p) { return split_chunk_ws_bytes(p); }

int launch_split_chunk(const FwdParams &p, cudaStream_t s) {
    auto al16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!split_chunk_covers(p) || !al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.out) ||
        (p.final_state && !al16(p.final_state)))
        return 1;
    const int BH = p.B * p.H, nch = (p.L + CH - 1) / CH;
    SplitMaps maps;
    if (!make_map(&maps.q, p.q, BH, p.L) || !make_map(&maps.k, p.k, BH, p.L) || !make_map(&maps.v, p.v, BH, p.L))
        return 1;
    void *ws = nullptr;
    bool owned = false;
    const size_t units = (size_t)BH * nch;
    const int wrc = ws_acquire(p.ws_given, p.ws, p.ws_bytes, split_chunk_ws_bytes(p), s, &ws, &owned);
    if (wrc) return wrc;
    uint8_t *img = static_cast<uint8_t *>(ws);
    float *gc = reinterpret_cast<float *>(img + units * IMG);
    static bool attrs_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs_set[dev]) {
        cudaFuncSetAttribute(chunk_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L_SMEM);
        cudaFuncSetAttribute(chunk_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_SMEM);
        if (dev >= 0 && dev < 64) attrs_set[dev] = true;
    }
    chunk_local_kernel<<<(unsigned)std::min<size_t>(units, (size_t)2 * sm_count()), NTH1, L_SMEM, s>>>(p, maps, img, gc);
    // the chain kernel as a programmatic dependent launch (see griddepcontrol in both kernels)
    if (cudaGetLastError() != cudaSuccess) {
        ws_release(ws, owned, s);
        return -7;  // FALCON_ERR_LAUNCH
    }
    const int crc = launch_chain_images(p, img, gc, s);
    ws_release(ws, owned, s);
    return crc;
}

int launch_chain_images(const FwdParams &p, const uint8_t *img, const float *gc, cudaStream_t s) {
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaFuncSetAttribute(chunk_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_SMEM);
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.B * p.H);
    cfg.blockDim = dim3(NTH2);
    cfg.dynamicSmemBytes = S_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, chunk_chain_kernel, p, img, gc);
    return cudaGetLastError() == cudaSuccess ? 0 : -7;  // FALCON_ERR_LAUNCH
}
#ifdef FALCON_TC_DEBUG
extern "C" int falcon_split_debug_timer_set(long long *ptr) {
    return cudaMemcpyToSymbol(g_split_tim, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : -1;
}
#endif

unsigned int split_wait_timeouts() {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_split_wait_timeouts, sizeof(v));
    return v;
}

}  // namespace falcon
