// k_chunk_tc.cu -- chunk-parallel forward on the tcgen05 tensor cores, bf16
// inputs, fp32 accumulation and state (Falcon-1 and Falcon-1A, d_k = d_v =
// 64, chunk 64).
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
//   O     = Qt S^T + O0,   S_end = g_C S - S Phi' + B.
// Only the last line depends on S, and it is one tensor-core product per
// chunk: [S;0] [Qt ; -Phi'^T]^T accumulated onto [O0^T | B], which yields the
// chunk's outputs (transposed) and the state increment together.  Every decay
// factor is a difference of cumulative logs, hence <= 1.
//
// Every tcgen05 operand is K-major (rows of 128 bytes, 128-byte swizzle), so
// each product is laid out as D = A B^T with both operands stored row-wise;
// the transposed operands are made by the tensor core itself (A = [.; I]):
//   G1  A=[X;Q]           B=X            -> A (lanes 0-63), P (lanes 64-127)
//   GT  A=[.;I] B=X -> X^T (lanes 64-127);  A=[I;.] B=Y -> Y^T (lanes 0-63)
//       CUDA cores: M, P o Dm, T = (I+M)^{-1} (16x16 blocked inversion, fp32)
//   G2  A=[Y^T;(D_a X)^T] B=T            -> U0^T (lanes 0-63), W^T (64-127)
//   G3  A=[P o Dm;(D_w X)^T] B=W^T       -> (P o Dm)W (0-63), Phi'^T (64-127)
//   G4  A=[U0^T;W^T]      B=[P o Dm;(D_w X)^T] -> [O0^T | B] (lanes 0-63)
//   G5  A=[S;0]           B=[Qt;-Phi'^T], accumulating onto G4
//                                        -> [O^T | B - S Phi'] (lanes 0-63)
// One thread block per (b,h), 256 threads; warp w reads tensor-memory lanes
// 32(w%4)..32(w%4)+31, and the two warps of a lane quarter split the columns.  The next chunk's q, k, v are prefetched with cp.async.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

constexpr int CH = 64;  // chunk
constexpr int DD = 64;  // d_k = d_v
constexpr int NTH = 256;
constexpr int ISSUER = 128;  // the thread that issues every tensor-core MMA (warp 4)
constexpr uint32_t TMEM_COLS = 512;
// accumulator columns (each starts at a multiple of 128)
constexpr uint32_t COL_G1 = 0, COL_G2 = 128, COL_G3 = 256, COL_G45 = 384;
constexpr uint32_t COL_S = 64;  // fp32 state S, rows j in lanes 0-63
constexpr uint32_t COL_XT = 192, COL_YT = 320;  // X^T in lanes 64-127, Y^T in lanes 0-63

// shared-memory byte offsets; operand tiles are 64 rows x 128 B (8 KB),
// 1024-byte aligned, 128-row operands are two consecutive tiles
constexpr uint32_t TILE = 8192;
constexpr uint32_t OFF_XQ0 = 0;            // [X;Q], buffer 0
constexpr uint32_t OFF_XQ1 = 2 * TILE;     // [X;Q], buffer 1
constexpr uint32_t OFF_XT = 4 * TILE;      // [Y^T ; (D_a X)^T]
constexpr uint32_t OFF_TA = 6 * TILE;      // T
constexpr uint32_t OFF_WUT = 7 * TILE;     // [U0^T ; W^T]
constexpr uint32_t OFF_A3 = 9 * TILE;      // [P o Dm ; (D_w X)^T]
constexpr uint32_t OFF_B5 = 11 * TILE;     // [Qt ; -Phi'^T]
constexpr uint32_t OFF_SA = 13 * TILE;     // [S ; 0]
constexpr uint32_t OFF_KR = 15 * TILE;     // raw keys (prefetch)
constexpr uint32_t OFF_VR0 = 16 * TILE;    // raw values, buffer 0
constexpr uint32_t OFF_VR1 = 17 * TILE;    // raw values, buffer 1
constexpr uint32_t OFF_IDT = 18 * TILE;    // bf16 identity (the tile before it pads A to 128 rows)
constexpr uint32_t OFF_MF = 19 * TILE;     // fp32 M [64][68]
// row stride 68 floats: float4 row stores and the m16n8k8 fragment loads
// below are both free of bank conflicts
constexpr uint32_t LDF = 68;
constexpr uint32_t OFF_TF = OFF_MF + 64 * LDF * 4;  // fp32 T [64][68]
constexpr uint32_t LDZ = 36;
constexpr uint32_t OFF_ZF = OFF_TF + 64 * LDF * 4;  // fp32 scratch [32][36]
constexpr uint32_t OFF_VEC = OFF_ZF + 32 * LDZ * 4;  // per-token vectors
constexpr uint32_t OFF_BAR = OFF_VEC + 8 * 64 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;  // + alignment slack

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



__device__ unsigned int g_tc_wait_timeouts;

#ifdef FALCON_TC_DEBUG
__device__ volatile int *g_stage;
__device__ float *g_dbg;
#define STAGE(sv)                                                      \
    do {                                                               \
        if (g_stage && threadIdx.x == 0) {                             \
            g_stage[blockIdx.x] = (sv);                                \
            __threadfence_system();                                    \
        }                                                              \
    } while (0)
__device__ long long *g_tim;
#define TIM(c, slot)                                                                \
    do {                                                                            \
        if (g_tim && blockIdx.x == 0 && threadIdx.x == 0 && (c) < 64)               \
            g_tim[(c) * 16 + (slot)] = clock64();                                   \
    } while (0)
#define TIMT(c, slot, th)                                                           \
    do {                                                                            \
        if (g_tim && blockIdx.x == 0 && threadIdx.x == (th) && (c) < 64)            \
            g_tim[(c) * 16 + (slot)] = clock64();                                   \
    } while (0)
#define TIMX(c, slot)                                                               \
    do {                                                                            \
        if ((c) == 5 && g_tim && blockIdx.x == 0 && (threadIdx.x == 0 || threadIdx.x == 64)) \
            g_tim[64 * 16 + (threadIdx.x ? 32 : 0) + (slot)] = clock64();           \
    } while (0)
#define DBG_ON(c) (g_dbg != nullptr && blockIdx.x == 0 && (c) < 2)
#define DBG(c, off) (g_dbg + (size_t)(c) * 50000 + (off))
#else
#define STAGE(sv)
#define TIM(c, slot)
#define TIMT(c, slot, th)
#define TIMX(c, slot)
#endif

// Bounded wait on an MMA-completion or TMA-arrival barrier: two seconds at most.
__device__ __forceinline__ bool wait_mma(uint64_t *bar, uint32_t parity) {
    return tc::mbar_wait_timeout(bar, parity, 2000000000ull);
}

// Tensor maps of q, k, v: 3-D [B*H][L][64] bf16, boxes of 64 x 64, 128-byte swizzle.
struct TcMaps {
    CUtensorMap q, k, v;
};

// TMA prefetch of chunk c0 (one thread): raw keys (row t <- key c0+t-1; the
// key before the sequence start and rows past its end read as zeros),
// queries and values, 24 KB completing on `bar`.
__device__ __forceinline__ void prefetch_tma(const TcMaps &m, int bh, int c0, uint32_t base, uint32_t off_q,
                                             uint32_t off_v, uint64_t *bar) {
    tc::mbar_arrive_expect_tx(bar, 3 * TILE);
    tc::tma_load_3d(base + OFF_KR, &m.k, 0, c0 - 1, bh, bar);
    tc::tma_load_3d(base + off_q, &m.q, 0, c0, bh, bar);
    tc::tma_load_3d(base + off_v, &m.v, 0, c0, bh, bar);
}

// D = A B^T over K = 64 (four K=16 slices), both operands K-major and
// 128-byte swizzled; M = 128, N = 64 or 128.
__device__ __forceinline__ void issue_gemm(uint32_t d_tmem, uint32_t a_saddr, uint32_t b_saddr, int N,
                                           bool accumulate) {
    const uint32_t idesc = tc::idesc_bf16(128, N, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = tc::sdesc_sw128(a_saddr + kk * 32, 16, 1024);
        const uint64_t bd = tc::sdesc_sw128(b_saddr + kk * 32, 16, 1024);
        tc::mma_bf16(d_tmem, ad, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

// 64 fp32 columns of this thread's tensor-memory lane.



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

}  // namespace

__global__ void __launch_bounds__(NTH, 1) chunk_tc_kernel(FwdParams p, const __grid_constant__ TcMaps maps) {
    extern __shared__ uint8_t smem_raw[];
    // align the operand tiles to 1024 bytes of the shared address space
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = tc::smem_u32(sm);
    float *Mf = reinterpret_cast<float *>(sm + OFF_MF);
    float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
    float *Zf = reinterpret_cast<float *>(sm + OFF_ZF);
    float *vec = reinterpret_cast<float *>(sm + OFF_VEC);
    float *v_sqn = vec, *v_eta = vec + 64, *v_G = vec + 128, *v_gm1 = vec + 192, *v_gt = vec + 256,
          *v_w = vec + 320, *v_beta = vec + 384;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);       // MMA completion
    uint64_t *tbar = reinterpret_cast<uint64_t *>(sm + OFF_BAR + 16); // TMA arrival
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // tensor-memory lane quarter of this warp, and which half of a 64-column
    // accumulator it handles (two warps share each lane quarter)
    const int quarter = warp & 3, chalf = warp >> 2;
    const int row = quarter * 32 + lane;  // accumulator row this thread reads
    const bool reg = p.variant == F1;
    const int bh = blockIdx.x, h = bh % p.H;
    const int L = p.L;
    const float lam = p.lambda[h];
    const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(p.beta) + (size_t)bh * L;
    __nv_bfloat16 *ko = static_cast<__nv_bfloat16 *>(p.out) + (size_t)bh * L * DD;

    // zero: [S;0] (S_0 = 0 and the padding half), the (D_a X)^T half of XT
    // (stays zero for the inner-product family) and -Phi'^T (likewise)
    for (int i = tid; i < (int)(TILE / 16); i += NTH) {
        const uint4 z = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4 *>(sm + OFF_SA)[i] = z;
        reinterpret_cast<uint4 *>(sm + OFF_SA + TILE)[i] = z;
        reinterpret_cast<uint4 *>(sm + OFF_XT + TILE)[i] = z;
        reinterpret_cast<uint4 *>(sm + OFF_B5 + TILE)[i] = z;
    }
    // identity operand (bf16 1.0 = 0x3F80 on the diagonal)
    for (int i = tid; i < 64 * 8; i += NTH) {
        const int r = i >> 3, c16 = i & 7;
        uint4 u = make_uint4(0, 0, 0, 0);
        if ((r >> 3) == c16) {
            const uint32_t one = 0x3F80u << (16 * (r & 1));
            const int word = (r & 7) >> 1;
            if (word == 0) u.x = one; else if (word == 1) u.y = one; else if (word == 2) u.z = one; else u.w = one;
        }
        *reinterpret_cast<uint4 *>(sm + OFF_IDT + tc::sw128(r, c16)) = u;
    }
    // T's strictly-upper blocks are read as zeros by the block products
    for (int i = tid; i < 64 * (int)LDF; i += NTH) Tf[i] = 0.f;
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_init(tbar, 1);
        tc::fence_mbar_init();
    }
    if (tid == NTH - 32) {
        tc::prefetch_tmap(&maps.q);
        tc::prefetch_tmap(&maps.k);
        tc::prefetch_tmap(&maps.v);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    __syncthreads();
    if (tid == NTH - 32) prefetch_tma(maps, bh, 0, sbase, OFF_XQ0 + TILE, OFF_VR0, tbar);
    bool tma_inflight = true;
    // beta of the next chunk travels as raw bf16 and is converted only when it
    // is stored a chunk later, so no warp waits on the global load
    __nv_bfloat16 beta_next = __float2bfloat16_rn(0.f);
    if (tid < 64 && tid < L) beta_next = kb[tid];
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(quarter * 32) << 16);  // this warp's lanes
    STAGE(1);
    if (quarter < 2) {  // S_0 = 0 (fp32 state, rows j in lanes 0-63)
        float z16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z16[i] = 0.f;
        tc::tmem_st16(tlane + COL_S + chalf * 32, z16);
        tc::tmem_st16(tlane + COL_S + chalf * 32 + 16, z16);
        tc::tmem_wait_st();
    }

    uint32_t phase = 0, tphase = 0;
    bool ok = true;
    const int nchunks = (L + CH - 1) / CH;
    const float4 *G4 = reinterpret_cast<const float4 *>(v_G);
    const float4 *E4 = reinterpret_cast<const float4 *>(v_eta);

    for (int c = 0; c < nchunks && ok; ++c) {
        const int c0 = c * CH;
        const int cur = c & 1;
        const uint32_t off_xq = cur ? OFF_XQ1 : OFF_XQ0;
        uint8_t *tX = sm + off_xq, *tQ = sm + off_xq + TILE;

        ok = wait_mma(tbar, tphase);  // this chunk's q, k, v have landed
        tphase ^= 1;
        tma_inflight = false;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        STAGE(10 * c + 2);
        TIM(c, 0);

        // ---- samples x_t = phi(k_{t-1}): four threads per row t
        {
            const int r = tid >> 2, part = tid & 3;
            float xr[16];
            float ss = 0.f;
#pragma unroll
            for (int c16 = 0; c16 < 2; ++c16) {
                unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_KR + tc::sw128(r, part * 2 + c16)), &xr[c16 * 8]);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss += xr[c16 * 8 + e] * xr[c16 * 8 + e];
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                xr[e] *= inv;
                sq += xr[e] * xr[e];
            }
            sq += __shfl_xor_sync(0xffffffffu, sq, 1);
            sq += __shfl_xor_sync(0xffffffffu, sq, 2);
#pragma unroll
            for (int c16 = 0; c16 < 2; ++c16)
                *reinterpret_cast<uint4 *>(tX + tc::sw128(r, part * 2 + c16)) = pack8(&xr[c16 * 8]);
            if (part == 0) v_sqn[r] = sq;
            if (tid < 64) v_beta[tid] = __bfloat162float(beta_next);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        TIM(c, 1);
        // ---- G1 [X;Q] X^T -> A, P and GT [.;I] X^T, [.;I] Y^T -> X^T, Y^T; they
        //      depend only on the samples and run while the steps are computed
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_gemm(tbase + COL_G1, sbase + off_xq, sbase + off_xq, 64, false);
            issue_gemm(tbase + COL_XT, sbase + OFF_IDT - TILE, sbase + off_xq, 64, false);
            issue_gemm(tbase + COL_YT, sbase + OFF_IDT, sbase + (cur ? OFF_VR1 : OFF_VR0), 64, false);
            tc::mma_commit(bar);
        }
        TIMT(c, 12, ISSUER);
        // raw keys consumed: prefetch the next chunk (beta into a register)
        if (c + 1 < nchunks) {
            if (tid == NTH - 32)
                prefetch_tma(maps, bh, c0 + CH, sbase, (cur ? OFF_XQ0 : OFF_XQ1) + TILE, cur ? OFF_VR0 : OFF_VR1,
                             tbar);
            TIMT(c, 13, NTH - 32);
            tma_inflight = true;
            beta_next = __float2bfloat16_rn(0.f);
            if (tid < 64 && c0 + CH + tid < L) beta_next = kb[c0 + CH + tid];
        }
        TIM(c, 10);

        // ---- steps, log decays and their chunk-local cumulative sums (warp 0,
        //      tokens 2l and 2l+1 on lane l)
        if (warp == 0) {
            const int t0 = 2 * lane;
            // eta = beta / (eps + n) (0 for an empty sample), alpha = max(1 - eta lambda, 2^-20)
            const float n0 = v_sqn[t0], n1 = v_sqn[t0 + 1];
            const float eta0 = n0 > 0.f ? __fdividef(v_beta[t0], p.eps + n0) : 0.f;
            const float eta1 = n1 > 0.f ? __fdividef(v_beta[t0 + 1], p.eps + n1) : 0.f;
            const float al0 = fmaxf(1.f - eta0 * lam, kAlphaFloor), al1 = fmaxf(1.f - eta1 * lam, kAlphaFloor);
            const float la0 = __logf(al0), la1 = __logf(al1);
            float run = la0 + la1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run += y;
            }
            const float G1v = run, G0v = run - la1, Gm = run - la0 - la1;  // G_{t0+1}, G_{t0}, G_{t0-1}
            const float GC = __shfl_sync(0xffffffffu, run, 31);
            v_eta[t0] = eta0;
            v_eta[t0 + 1] = eta1;
            v_G[t0] = G0v;
            v_G[t0 + 1] = G1v;
            v_gm1[t0] = __expf(Gm);
            v_gm1[t0 + 1] = __expf(G0v);
            v_gt[t0] = __expf(G0v);
            v_gt[t0 + 1] = __expf(G1v);
            v_w[t0] = __expf(GC - G0v) * eta0;
            v_w[t0 + 1] = __expf(GC - G1v) * eta1;
        }
        TIMT(c, 11, 0);
        __syncthreads();
        STAGE(10 * c + 3);
        TIM(c, 2);
        const float gC = __expf(v_G[63]);

        ok = wait_mma(bar, phase);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        STAGE(10 * c + 4);
        TIM(c, 3);
        {
            // rows 0-63: M[t][s] = (g_{t-1}/g_s) eta_s A[t][s] for s < t (fp32);
            // rows 64-127: (P o Dm)[t][s] = (g_t/g_s) eta_s P[t][s] for s <= t (bf16).
            // Branch-free: every exponent is computed (argument clamped to <= 0)
            // and masked afterwards, so the 16 chains of a slice overlap.
            const bool mrow = quarter < 2;
            const int t = mrow ? row : row - 64;
            const float gref = mrow ? (t > 0 ? v_G[t - 1] : 0.f) : v_G[t];
            const int tlim = mrow ? t : t + 1;  // s < tlim
            const bool active = mrow ? reg : true;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16], gs[16], es[16];
                tc::tmem_ld16(tlane + COL_G1 + cs * 16, v);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 g = G4[cs * 4 + q], e = E4[cs * 4 + q];
                    gs[q * 4 + 0] = g.x; gs[q * 4 + 1] = g.y; gs[q * 4 + 2] = g.z; gs[q * 4 + 3] = g.w;
                    es[q * 4 + 0] = e.x; es[q * 4 + 1] = e.y; es[q * 4 + 2] = e.z; es[q * 4 + 3] = e.w;
                }
                tc::tmem_wait_ld();
                float m[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float x = __expf(fminf(gref - gs[i], 0.f)) * es[i] * v[i];
                    m[i] = (active && cs * 16 + i < tlim) ? x : 0.f;
                }
                if (mrow) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4 *>(Mf + t * LDF + cs * 16 + q * 4) =
                            make_float4(m[q * 4], m[q * 4 + 1], m[q * 4 + 2], m[q * 4 + 3]);
                    // Y^T row n = t -> XT[n]
                    float yt[16];
                    tc::tmem_ld16(tlane + COL_YT + cs * 16, yt);
                    tc::tmem_wait_ld();
                    *reinterpret_cast<uint4 *>(sm + OFF_XT + tc::sw128(t, cs * 2)) = pack8(&yt[0]);
                    *reinterpret_cast<uint4 *>(sm + OFF_XT + tc::sw128(t, cs * 2 + 1)) = pack8(&yt[8]);
                } else {
                    *reinterpret_cast<uint4 *>(sm + OFF_A3 + tc::sw128(t, cs * 2)) = pack8(&m[0]);
                    *reinterpret_cast<uint4 *>(sm + OFF_A3 + tc::sw128(t, cs * 2 + 1)) = pack8(&m[8]);
                    // transposed rows n = t: (D_w X)^T -> A3[64+n], (D_a X)^T -> XT[64+n] (regression)
                    float xt[16], ws[16], as[16];
                    tc::tmem_ld16(tlane + COL_XT + cs * 16, xt);
                    const float4 *W4 = reinterpret_cast<const float4 *>(v_w);
                    const float4 *A4 = reinterpret_cast<const float4 *>(v_gm1);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 w = W4[cs * 4 + q], a = A4[cs * 4 + q];
                        ws[q * 4 + 0] = w.x; ws[q * 4 + 1] = w.y; ws[q * 4 + 2] = w.z; ws[q * 4 + 3] = w.w;
                        as[q * 4 + 0] = a.x; as[q * 4 + 1] = a.y; as[q * 4 + 2] = a.z; as[q * 4 + 3] = a.w;
                    }
                    tc::tmem_wait_ld();
                    float o8[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) o8[i] = xt[i] * ws[i];
                    *reinterpret_cast<uint4 *>(sm + OFF_A3 + TILE + tc::sw128(t, cs * 2)) = pack8(&o8[0]);
                    *reinterpret_cast<uint4 *>(sm + OFF_A3 + TILE + tc::sw128(t, cs * 2 + 1)) = pack8(&o8[8]);
                    if (reg) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) o8[i] = xt[i] * as[i];
                        *reinterpret_cast<uint4 *>(sm + OFF_XT + TILE + tc::sw128(t, cs * 2)) = pack8(&o8[0]);
                        *reinterpret_cast<uint4 *>(sm + OFF_XT + TILE + tc::sw128(t, cs * 2 + 1)) = pack8(&o8[8]);
                    }
                }
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        STAGE(10 * c + 5);
        TIM(c, 4);

        uint32_t a4 = sbase + OFF_XT;  // A of G4: [U0^T; W^T], or [Y^T; 0] for the A family
        if (reg) {
            // ---- T = (I + M)^{-1}.  Diagonal 16x16 blocks by forward
            //      substitution (warp b, lane = column); the off-diagonal
            //      blocks by T_ij = -T_ii (M_i. T_.j) with TF32 warp MMAs.
            if (warp < 4 && lane < 16) {
                const int b0 = warp * 16, j = lane;
                float tcol[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float *mr = Mf + (b0 + i) * LDF + b0;
                    float acc0 = (i == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                    for (int s = 0; s + 1 < i; s += 2) {
                        acc0 -= mr[s] * tcol[s];
                        acc1 -= mr[s + 1] * tcol[s + 1];
                    }
                    if (i & 1) acc0 -= mr[i - 1] * tcol[i - 1];
                    tcol[i] = acc0 + acc1;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) Tf[(b0 + i) * LDF + b0 + j] = tcol[i];
            }
            __syncthreads();
            if (warp < 4) {  // blocks (1,0) [warps 0,1] and (3,2) [warps 2,3]; warp = 8 columns
                const int pb = warp >> 1, nt = warp & 1;
                const int r0 = pb ? 48 : 16, q0 = pb ? 32 : 0;
                float *zw = Zf + warp * 16 * 8;  // this warp's 16 x 8 scratch
                float c4[4];
                warp_gemm_16x8<16>(Mf + r0 * LDF + q0, LDF, Tf + q0 * LDF + q0 + nt * 8, LDF, c4);
                warp_store_16x8(zw, 8, c4, 1.f);
                __syncwarp();
                warp_gemm_16x8<16>(Tf + r0 * LDF + r0, LDF, zw, 8, c4);
                warp_store_16x8(Tf + r0 * LDF + q0 + nt * 8, LDF, c4, -1.f);
            }
            __syncthreads();
            // 32x32 block (rows 32-63, cols 0-31); warp = one 16x8 tile
            const int rb = warp >> 2, cb = (warp >> 1) & 1, nt = warp & 1;
            {   // Z = M_HL T_LL
                float c4[4];
                warp_gemm_16x8<32>(Mf + (32 + rb * 16) * LDF, LDF, Tf + cb * 16 + nt * 8, LDF, c4);
                warp_store_16x8(Zf + rb * 16 * LDZ + cb * 16 + nt * 8, LDZ, c4, 1.f);
            }
            __syncthreads();
            {   // T_HL = -T_HH Z
                float c4[4];
                warp_gemm_16x8<32>(Tf + (32 + rb * 16) * LDF + 32, LDF, Zf + cb * 16 + nt * 8, LDZ, c4);
                warp_store_16x8(Tf + (32 + rb * 16) * LDF + cb * 16 + nt * 8, LDF, c4, -1.f);
            }
            __syncthreads();
            {   // T (lower triangle) to bf16: thread = (row, 16 columns)
                const int r = tid >> 2, part = tid & 3;
#pragma unroll
                for (int c16 = 0; c16 < 2; ++c16) {
                    float t8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = part * 16 + c16 * 8 + e;
                        t8[e] = s <= r ? Tf[r * LDF + s] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(sm + OFF_TA + tc::sw128(r, part * 2 + c16)) = pack8(t8);
                }
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            STAGE(10 * c + 6);
            TIM(c, 5);

            // ---- G2: [Y^T;(D_a X)^T] T^T -> U0^T (lanes 0-63), W^T (lanes 64-127)
            if (tid == ISSUER) {
                tc::fence_after_sync();
                issue_gemm(tbase + COL_G2, sbase + OFF_XT, sbase + OFF_TA, 64, false);
                tc::mma_commit(bar);
            }
            ok = wait_mma(bar, phase);
            phase ^= 1;
            ok = __syncthreads_and(ok);
            if (!ok) break;
            tc::fence_after_sync();
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16];
                tc::tmem_ld16(tlane + COL_G2 + cs * 16, v);
                tc::tmem_wait_ld();
                *reinterpret_cast<uint4 *>(sm + OFF_WUT + tc::sw128(row, cs * 2)) = pack8(&v[0]);
                *reinterpret_cast<uint4 *>(sm + OFF_WUT + tc::sw128(row, cs * 2 + 1)) = pack8(&v[8]);
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            STAGE(10 * c + 7);
            TIM(c, 6);

            // ---- G3: [P o Dm;(D_w X)^T] W -> (P o Dm) W (lanes 0-63), Phi'^T (lanes 64-127)
            if (tid == ISSUER) {
                tc::fence_after_sync();
                issue_gemm(tbase + COL_G3, sbase + OFF_A3, sbase + OFF_WUT + TILE, 64, false);
                tc::mma_commit(bar);
            }
            ok = wait_mma(bar, phase);
            phase ^= 1;
            ok = __syncthreads_and(ok);
            if (!ok) break;
            tc::fence_after_sync();
            {
                const bool qrow = quarter < 2;
                const float g = qrow ? v_gt[row] : -1.f;
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    const int cs = chalf * 2 + k2;
                    float v[16];
                    tc::tmem_ld16(tlane + COL_G3 + cs * 16, v);
                    tc::tmem_wait_ld();
                    if (qrow) {  // Qt = D_g Q - (P o Dm) W
                        float q8[8];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            unpack8(*reinterpret_cast<const uint4 *>(tQ + tc::sw128(row, cs * 2 + hh)), q8);
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[hh * 8 + i] = g * q8[i] - v[hh * 8 + i];
                        }
                        *reinterpret_cast<uint4 *>(sm + OFF_B5 + tc::sw128(row, cs * 2)) = pack8(&v[0]);
                        *reinterpret_cast<uint4 *>(sm + OFF_B5 + tc::sw128(row, cs * 2 + 1)) = pack8(&v[8]);
                    } else {  // -Phi'^T
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = -v[i];
                        *reinterpret_cast<uint4 *>(sm + OFF_B5 + TILE + tc::sw128(row - 64, cs * 2)) = pack8(&v[0]);
                        *reinterpret_cast<uint4 *>(sm + OFF_B5 + TILE + tc::sw128(row - 64, cs * 2 + 1)) =
                            pack8(&v[8]);
                    }
                }
            }
            a4 = sbase + OFF_WUT;
        } else if (quarter < 2) {  // inner-product family: Qt = D_g Q
            const float g = v_gt[row];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float q8[8];
                unpack8(*reinterpret_cast<const uint4 *>(tQ + tc::sw128(row, chalf * 4 + cc)), q8);
#pragma unroll
                for (int i = 0; i < 8; ++i) q8[i] *= g;
                *reinterpret_cast<uint4 *>(sm + OFF_B5 + tc::sw128(row, chalf * 4 + cc)) = pack8(q8);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        STAGE(10 * c + 8);
        TIM(c, 7);

        // ---- G4 then G5 (the chain) into one accumulator:
        //      [U0^T;W^T] [P o Dm;(D_w X)^T]^T + [S;0] [Qt;-Phi'^T]^T
        if (tid == ISSUER) {
            tc::fence_after_sync();
            issue_gemm(tbase + COL_G45, a4, sbase + OFF_A3, 128, false);
            issue_gemm(tbase + COL_G45, sbase + OFF_SA, sbase + OFF_B5, 128, true);
            tc::mma_commit(bar);
        }
        ok = wait_mma(bar, phase);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        TIM(c, 8);
        if (quarter < 2) {
            const int j = row;
            const int nt = min(CH, L - c0);
            // outputs: O^T[j][t] -> out[c0 + t][j], this warp's 32 tokens
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float v[16];
                tc::tmem_ld16(tlane + COL_G45 + cs * 16, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (cs * 16 + i < nt) ko[(size_t)(c0 + cs * 16 + i) * DD + j] = __float2bfloat16_rn(v[i]);
            }
            // state: S_end = g_C S + (B - S Phi'), fp32 in tensor memory, bf16 copy for the next chain MMA
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cs = chalf * 2 + k2;
                float ds[16], sv[16];
                tc::tmem_ld16(tlane + COL_G45 + 64 + cs * 16, ds);
                tc::tmem_ld16(tlane + COL_S + cs * 16, sv);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[i] = gC * sv[i] + ds[i];
                tc::tmem_st16(tlane + COL_S + cs * 16, sv);
                *reinterpret_cast<uint4 *>(sm + OFF_SA + tc::sw128(j, cs * 2)) = pack8(&sv[0]);
                *reinterpret_cast<uint4 *>(sm + OFF_SA + tc::sw128(j, cs * 2 + 1)) = pack8(&sv[8]);
            }
            tc::tmem_wait_st();
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        STAGE(10 * c + 9);
        TIM(c, 9);
    }

    STAGE(ok ? 9999 : -2);
    if (!ok && tid == 0) atomicAdd(&g_tc_wait_timeouts, 1u);
    if (ok && p.final_state && quarter < 2) {
        float *fs = p.final_state + ((size_t)bh * DD + row) * DD;
        tc::fence_after_sync();
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
            const int cs = chalf * 2 + k2;
            float sv[16];
            tc::tmem_ld16(tlane + COL_S + cs * 16, sv);
            tc::tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4 *>(fs + cs * 16 + q * 4) =
                    make_float4(sv[q * 4], sv[q * 4 + 1], sv[q * 4 + 2], sv[q * 4 + 3]);
        }
    }
    // a prefetch abandoned by an early exit must land before the block leaves
    if (tma_inflight && !ok) (void)wait_mma(tbar, tphase);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, TMEM_COLS);
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

int launch_tc_chunk(const FwdParams &p, cudaStream_t s) {
    const bool shape_ok = (p.variant == F1 || p.variant == F1A) && p.dk == DD && p.dv == DD && p.chunk == CH &&
                          p.pairing == 0 && p.phi == 0;
    auto al16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!shape_ok || !al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.out) ||
        (p.final_state && !al16(p.final_state)))
        return 1;
    TcMaps maps;
    const int BH = p.B * p.H;
    if (!make_map(&maps.q, p.q, BH, p.L) || !make_map(&maps.k, p.k, BH, p.L) || !make_map(&maps.v, p.v, BH, p.L))
        return 1;
    cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    chunk_tc_kernel<<<BH, NTH, SMEM_BYTES, s>>>(p, maps);
    return 0;
}

#ifdef FALCON_TC_DEBUG
extern "C" int *falcon_tc_debug_stage_alloc(int n) {
    int *h = nullptr, *d = nullptr;
    if (cudaHostAlloc((void **)&h, sizeof(int) * n, cudaHostAllocMapped) != cudaSuccess) return nullptr;
    for (int i = 0; i < n; ++i) h[i] = 0;
    if (cudaHostGetDevicePointer((void **)&d, h, 0) != cudaSuccess) return nullptr;
    if (cudaMemcpyToSymbol(g_stage, &d, sizeof(d)) != cudaSuccess) return nullptr;
    return h;
}
extern "C" int falcon_tc_debug_timer_set(long long *ptr) {
    return cudaMemcpyToSymbol(g_tim, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : -1;
}
extern "C" int falcon_tc_debug_set(float *ptr) {
    return cudaMemcpyToSymbol(g_dbg, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : -1;
}
#endif

unsigned int tc_wait_timeouts() {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_tc_wait_timeouts, sizeof(v));
    return v;
}

}  // namespace falcon
