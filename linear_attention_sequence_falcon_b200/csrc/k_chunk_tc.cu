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
// each product is laid out as D = A B^T with both operands stored row-wise:
//   G1  A=[X;Q]           B=X            -> A (lanes 0-63), P (lanes 64-127)
//       CUDA cores: M, P o Dm, T = (I+M)^{-1} (16x16 blocked inversion, fp32)
//   G2  A=[Y^T;(D_a X)^T] B=T            -> U0^T (lanes 0-63), W^T (64-127)
//   G3  A=[P o Dm;(D_w X)^T] B=W^T       -> (P o Dm)W (0-63), Phi'^T (64-127)
//   G4  A=[U0^T;W^T]      B=[P o Dm;(D_w X)^T] -> [O0^T | B] (lanes 0-63)
//   G5  A=[S;0]           B=[Qt;-Phi'^T], accumulating onto G4
//                                        -> [O^T | B - S Phi'] (lanes 0-63)
// One thread block per (b,h), 128 threads; warp w reads tensor-memory lanes
// 32w..32w+31.  The next chunk's q, k, v are prefetched with cp.async.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {

namespace {

constexpr int CH = 64;  // chunk
constexpr int DD = 64;  // d_k = d_v
constexpr int NTH = 128;
constexpr uint32_t TMEM_COLS = 512;
// accumulator columns (each starts at a multiple of 128)
constexpr uint32_t COL_G1 = 0, COL_G2 = 128, COL_G3 = 256, COL_G45 = 384;

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
constexpr uint32_t OFF_MF = 18 * TILE;     // fp32 M [64][65]
constexpr uint32_t LDF = 65;
constexpr uint32_t OFF_TF = OFF_MF + 64 * LDF * 4;  // fp32 T [64][65]
constexpr uint32_t OFF_ZF = OFF_TF + 64 * LDF * 4;  // fp32 scratch [32][33]
constexpr uint32_t OFF_VEC = OFF_ZF + 32 * 33 * 4;  // per-token vectors
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

// one bf16 element (row r, column col) of a 128-byte-swizzled tile
__device__ __forceinline__ void st_elem(uint8_t *tile, int r, int col, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(tile + tc::sw128(r, col >> 3) + (col & 7) * 2) = __float2bfloat16_rn(x);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
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
#define DBG_ON(c) (g_dbg != nullptr && blockIdx.x == 0 && (c) < 2)
#define DBG(c, off) (g_dbg + (size_t)(c) * 50000 + (off))
#else
#define STAGE(sv)
#endif

// Bounded wait on the MMA-completion barrier: about two seconds at most.
__device__ __forceinline__ bool wait_mma(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > 2000000000ull) return false;
    }
    return true;
}

// Prefetch chunk c0's raw keys (row t <- key c0+t-1), queries and values.
__device__ __forceinline__ void prefetch(const __nv_bfloat16 *kq, const __nv_bfloat16 *kk,
                                         const __nv_bfloat16 *kv, int L, int c0, uint32_t base,
                                         uint32_t off_q, uint32_t off_v) {
    for (int i = threadIdx.x; i < 3 * 64 * 8; i += NTH) {
        const int which = i / 512, r = (i / 8) % 64, c16 = i % 8;
        const int tok = c0 + r;
        if (which == 0) {
            const int kt = tok - 1;
            const bool ok = kt >= 0 && tok < L;
            cp_async16(base + OFF_KR + tc::sw128(r, c16), kk + (size_t)(ok ? kt : 0) * DD + c16 * 8, ok);
        } else {
            const bool ok = tok < L;
            const __nv_bfloat16 *src = which == 1 ? kq : kv;
            cp_async16(base + (which == 1 ? off_q : off_v) + tc::sw128(r, c16),
                       src + (size_t)(ok ? tok : 0) * DD + c16 * 8, ok);
        }
    }
    cp_async_commit();
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
__device__ __forceinline__ void tmem_row64(uint32_t tbase, int warp, uint32_t col, float (&v)[64]) {
    float a[32], b[32];
    const uint32_t addr = tbase + ((uint32_t)(warp * 32) << 16) + col;
    tc::tmem_ld32(addr, a);
    tc::tmem_ld32(addr + 32, b);
    tc::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        v[i] = a[i];
        v[32 + i] = b[i];
    }
}

__device__ __forceinline__ void store_row_bf16(uint8_t *tile, int r, const float (&v)[64], float scale = 1.f) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float t8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t8[e] = v[c * 8 + e] * scale;
        *reinterpret_cast<uint4 *>(tile + tc::sw128(r, c)) = pack8(t8);
    }
}

__device__ __forceinline__ void load_row_bf16(const uint8_t *tile, int r, float (&v)[64]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) unpack8(*reinterpret_cast<const uint4 *>(tile + tc::sw128(r, c)), &v[c * 8]);
}

}  // namespace

__global__ void __launch_bounds__(NTH, 1) chunk_tc_kernel(FwdParams p) {
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
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool reg = p.variant == F1;
    const int bh = blockIdx.x, h = bh % p.H;
    const int L = p.L;
    const float lam = p.lambda[h];
    const __nv_bfloat16 *kq = static_cast<const __nv_bfloat16 *>(p.q) + (size_t)bh * L * DD;
    const __nv_bfloat16 *kk = static_cast<const __nv_bfloat16 *>(p.k) + (size_t)bh * L * DD;
    const __nv_bfloat16 *kv = static_cast<const __nv_bfloat16 *>(p.v) + (size_t)bh * L * DD;
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
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    prefetch(kq, kk, kv, L, 0, sbase, OFF_XQ0 + TILE, OFF_VR0);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    STAGE(1);

    float Sreg[64];  // warps 0,1: row j = tid of S, fp32
#pragma unroll
    for (int i = 0; i < 64; ++i) Sreg[i] = 0.f;
    uint32_t phase = 0;
    bool ok = true;
    const int nchunks = (L + CH - 1) / CH;

    for (int c = 0; c < nchunks && ok; ++c) {
        const int c0 = c * CH;
        const int cur = c & 1;
        const uint32_t off_xq = cur ? OFF_XQ1 : OFF_XQ0;
        uint8_t *tX = sm + off_xq, *tQ = sm + off_xq + TILE;
        const uint8_t *tV = sm + (cur ? OFF_VR1 : OFF_VR0);

        cp_async_wait_all();
        __syncthreads();
        STAGE(10 * c + 2);

        // ---- samples x_t = phi(k_{t-1}): two threads per row t; Y^T from the raw values
        const int r = tid >> 1, half = tid & 1;
        float xr[32];
        {
            float ss = 0.f;
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                unpack8(*reinterpret_cast<const uint4 *>(sm + OFF_KR + tc::sw128(r, half * 4 + c16)), &xr[c16 * 8]);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss += xr[c16 * 8 + e] * xr[c16 * 8 + e];
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                xr[e] *= inv;
                sq += xr[e] * xr[e];
            }
            sq += __shfl_xor_sync(0xffffffffu, sq, 1);
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16)
                *reinterpret_cast<uint4 *>(tX + tc::sw128(r, half * 4 + c16)) = pack8(&xr[c16 * 8]);
            float yv[32];
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16)
                unpack8(*reinterpret_cast<const uint4 *>(tV + tc::sw128(r, half * 4 + c16)), &yv[c16 * 8]);
#pragma unroll
            for (int e = 0; e < 32; ++e) st_elem(sm + OFF_XT, half * 32 + e, r, yv[e]);  // Y^T
            if (half == 0) {
                v_sqn[r] = sq;
                v_beta[r] = (c0 + r < L) ? __bfloat162float(kb[c0 + r]) : 0.f;
            }
        }
        __syncthreads();
        // raw keys and values consumed: prefetch the next chunk
        if (c + 1 < nchunks)
            prefetch(kq, kk, kv, L, c0 + CH, sbase, (cur ? OFF_XQ0 : OFF_XQ1) + TILE, cur ? OFF_VR0 : OFF_VR1);

        // ---- steps, log decays and their chunk-local cumulative sums
        if (tid < 64) {
            float eta, alpha;
            step_and_decay(v_beta[tid], v_sqn[tid], p.eps, lam, eta, alpha);
            float la = __logf(alpha);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, la, o);
                if (lane >= o) la += y;
            }
            v_eta[tid] = eta;
            v_G[tid] = la;
        }
        __syncthreads();
        if (tid >= 32 && tid < 64) v_G[tid] += v_G[31];
        __syncthreads();
        if (tid < 64) {
            const float G = v_G[tid];
            v_gm1[tid] = __expf(tid > 0 ? v_G[tid - 1] : 0.f);
            v_gt[tid] = __expf(G);
            v_w[tid] = __expf(v_G[63] - G) * v_eta[tid];
        }
        __syncthreads();
        const float gC = __expf(v_G[63]);

        // ---- (D_a X)^T (regression) and (D_w X)^T, column r of each
        {
            const float ws = v_w[r], ga = v_gm1[r];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                st_elem(sm + OFF_A3 + TILE, half * 32 + e, r, xr[e] * ws);
                if (reg) st_elem(sm + OFF_XT + TILE, half * 32 + e, r, xr[e] * ga);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        STAGE(10 * c + 3);

        // ---- G1: [X;Q] X^T -> A (lanes 0-63), P (lanes 64-127)
        if (tid == 0) {
            tc::fence_after_sync();
            issue_gemm(tbase + COL_G1, sbase + off_xq, sbase + off_xq, 64, false);
            tc::mma_commit(bar);
        }
        ok = wait_mma(bar, phase);
        phase ^= 1;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        STAGE(10 * c + 4);
        {
            float v[64];
            tmem_row64(tbase, warp, COL_G1, v);
#ifdef FALCON_TC_DEBUG
            if (DBG_ON(c)) for (int i = 0; i < 64; ++i) DBG(c, (warp < 2 ? 0 : 4096) + (tid & 63) * 64 + i)[0] = v[i];
            if (DBG_ON(c) && tid < 64) for (int i = 0; i < 7; ++i) DBG(c, 49152 + i * 64 + tid)[0] = vec[i * 64 + tid];
#endif
            if (warp < 2) {
                const int t = tid;
                const float gp = t > 0 ? v_G[t - 1] : 0.f;
#pragma unroll
                for (int s = 0; s < 64; ++s)
                    Mf[t * LDF + s] = (reg && s < t) ? __expf(gp - v_G[s]) * v_eta[s] * v[s] : 0.f;
            } else {
                const int t = tid - 64;
                const float gt = v_G[t];
#pragma unroll
                for (int s = 0; s < 64; ++s) v[s] = s <= t ? v[s] * __expf(gt - v_G[s]) * v_eta[s] : 0.f;
                store_row_bf16(sm + OFF_A3, t, v);  // P o Dm
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        STAGE(10 * c + 5);

        uint32_t a4 = sbase + OFF_XT;  // A of G4: [U0^T; W^T], or [Y^T; 0] for the A family
        if (reg) {
            // ---- T = (I + M)^{-1}: 16x16 diagonal blocks by forward substitution
            if (lane < 16) {
                const int b0 = warp * 16, j = lane;
                float tcol[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
                    for (int s = 0; s < i; ++s) acc -= Mf[(b0 + i) * LDF + b0 + s] * tcol[s];
                    tcol[i] = acc;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) Tf[(b0 + i) * LDF + b0 + j] = tcol[i];
            }
            __syncthreads();
            // 16x16 off-diagonal blocks (1,0) and (3,2): T10 = -T11 (M10 T00)
            for (int idx = tid; idx < 512; idx += NTH) {
                const int pb = idx >> 8, i = (idx >> 4) & 15, j = idx & 15;
                const int r0 = pb ? 48 : 16, q0 = pb ? 32 : 0;
                float acc = 0.f;
                for (int s = j; s < 16; ++s) acc += Mf[(r0 + i) * LDF + q0 + s] * Tf[(q0 + s) * LDF + q0 + j];
                Zf[(pb * 16 + i) * 33 + j] = acc;
            }
            __syncthreads();
            for (int idx = tid; idx < 512; idx += NTH) {
                const int pb = idx >> 8, i = (idx >> 4) & 15, j = idx & 15;
                const int r0 = pb ? 48 : 16, q0 = pb ? 32 : 0;
                float acc = 0.f;
                for (int s = 0; s <= i; ++s) acc += Tf[(r0 + i) * LDF + r0 + s] * Zf[(pb * 16 + s) * 33 + j];
                Tf[(r0 + i) * LDF + q0 + j] = -acc;
            }
            __syncthreads();
            // 32x32 off-diagonal block: T_HL = -T_HH (M_HL T_LL)
            for (int idx = tid; idx < 1024; idx += NTH) {
                const int i = idx >> 5, j = idx & 31;
                float acc = 0.f;
                for (int s = j; s < 32; ++s) acc += Mf[(32 + i) * LDF + s] * Tf[s * LDF + j];
                Zf[i * 33 + j] = acc;
            }
            __syncthreads();
            for (int idx = tid; idx < 1024; idx += NTH) {
                const int i = idx >> 5, j = idx & 31;
                float acc = 0.f;
                for (int s = 0; s <= i; ++s) acc += Tf[(32 + i) * LDF + 32 + s] * Zf[s * 33 + j];
                Tf[(32 + i) * LDF + j] = -acc;
            }
            __syncthreads();
            {
                float t8[8];
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = half * 32 + c16 * 8 + e;
                        t8[e] = s <= r ? Tf[r * LDF + s] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(sm + OFF_TA + tc::sw128(r, half * 4 + c16)) = pack8(t8);
                }
            }
#ifdef FALCON_TC_DEBUG
            if (DBG_ON(c)) for (int i = tid; i < 4096; i += NTH) {
                DBG(c, 8192 + i)[0] = Mf[(i / 64) * LDF + i % 64];
                DBG(c, 12288 + i)[0] = Tf[(i / 64) * LDF + i % 64];
            }
#endif
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            STAGE(10 * c + 6);

            // ---- G2: [Y^T;(D_a X)^T] T^T -> U0^T (lanes 0-63), W^T (lanes 64-127)
            if (tid == 0) {
                tc::fence_after_sync();
                issue_gemm(tbase + COL_G2, sbase + OFF_XT, sbase + OFF_TA, 64, false);
                tc::mma_commit(bar);
            }
            ok = wait_mma(bar, phase);
            phase ^= 1;
            ok = __syncthreads_and(ok);
            if (!ok) break;
            tc::fence_after_sync();
            {
                float v[64];
                tmem_row64(tbase, warp, COL_G2, v);
#ifdef FALCON_TC_DEBUG
                if (DBG_ON(c)) for (int i = 0; i < 64; ++i) DBG(c, 16384 + tid * 64 + i)[0] = v[i];
#endif
                store_row_bf16(sm + OFF_WUT, tid, v);
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            STAGE(10 * c + 7);

            // ---- G3: [P o Dm;(D_w X)^T] W -> (P o Dm) W (lanes 0-63), Phi'^T (lanes 64-127)
            if (tid == 0) {
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
                float v[64];
                tmem_row64(tbase, warp, COL_G3, v);
#ifdef FALCON_TC_DEBUG
                if (DBG_ON(c)) for (int i = 0; i < 64; ++i) DBG(c, 24576 + tid * 64 + i)[0] = v[i];
#endif
                if (warp < 2) {  // Qt = D_g Q - (P o Dm) W
                    float qrow[64];
                    load_row_bf16(tQ, tid, qrow);
                    const float g = v_gt[tid];
#pragma unroll
                    for (int i = 0; i < 64; ++i) v[i] = g * qrow[i] - v[i];
                    store_row_bf16(sm + OFF_B5, tid, v);
                } else {  // -Phi'^T
                    store_row_bf16(sm + OFF_B5 + TILE, tid - 64, v, -1.f);
                }
            }
            a4 = sbase + OFF_WUT;
        } else if (warp < 2) {  // inner-product family: Qt = D_g Q
            float qrow[64];
            load_row_bf16(tQ, tid, qrow);
            store_row_bf16(sm + OFF_B5, tid, qrow, v_gt[tid]);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        STAGE(10 * c + 8);

        // ---- G4 then G5 (the chain) into one accumulator:
        //      [U0^T;W^T] [P o Dm;(D_w X)^T]^T + [S;0] [Qt;-Phi'^T]^T
        if (tid == 0) {
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
        {
            float v[64], e[64];
            tmem_row64(tbase, warp, COL_G45, v);       // O^T[j][t]
            tmem_row64(tbase, warp, COL_G45 + 64, e);  // (B - S Phi')[j][k]
#ifdef FALCON_TC_DEBUG
            if (DBG_ON(c) && warp < 2) for (int i = 0; i < 64; ++i) {
                DBG(c, 32768 + tid * 128 + i)[0] = v[i];
                DBG(c, 32768 + tid * 128 + 64 + i)[0] = e[i];
            }
#endif
            if (warp < 2) {
                const int j = tid;
                const int nt = min(CH, L - c0);
#pragma unroll
                for (int t = 0; t < 64; ++t)
                    if (t < nt) ko[(size_t)(c0 + t) * DD + j] = __float2bfloat16_rn(v[t]);
#pragma unroll
                for (int i = 0; i < 64; ++i) Sreg[i] = gC * Sreg[i] + e[i];
                store_row_bf16(sm + OFF_SA, j, Sreg);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        STAGE(10 * c + 9);
    }

    STAGE(ok ? 9999 : -2);
    if (!ok && tid == 0) atomicAdd(&g_tc_wait_timeouts, 1u);
    if (ok && p.final_state && warp < 2) {
        float *fs = p.final_state + ((size_t)bh * DD + tid) * DD;
#pragma unroll
        for (int c16 = 0; c16 < 16; ++c16)
            *reinterpret_cast<float4 *>(fs + c16 * 4) =
                make_float4(Sreg[c16 * 4], Sreg[c16 * 4 + 1], Sreg[c16 * 4 + 2], Sreg[c16 * 4 + 3]);
    }
    cp_async_wait_all();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, TMEM_COLS);
}

int launch_tc_chunk(const FwdParams &p, cudaStream_t s) {
    const bool shape_ok = (p.variant == F1 || p.variant == F1A) && p.dk == DD && p.dv == DD && p.chunk == CH &&
                          p.pairing == 0 && p.phi == 0;
    auto al16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    if (!shape_ok || !al16(p.q) || !al16(p.k) || !al16(p.v) || !al16(p.out) ||
        (p.final_state && !al16(p.final_state)))
        return 1;
    cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    chunk_tc_kernel<<<p.B * p.H, NTH, SMEM_BYTES, s>>>(p);
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
