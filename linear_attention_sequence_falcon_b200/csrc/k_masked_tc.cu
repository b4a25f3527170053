// k_masked_tc.cu -- the masked-parallel form of Falcon-1/1A and Falcon-3/3A (windows
// of 1-4 samples) on the tcgen05 tensor cores (bf16 inputs, d_k = d_v = 64, S_0 = 0).
//
// Method: "masked-parallel: every step at once through a causal mask" (page
// "Fast Weight Attention for Continual Learning", 方法/计算形式与数值稳定;
// page "Fast Weight Attention：用于持续学习的快速权重注意力", 核心方法 3).  With
// Gamma_t = sum_{r<=t} log alpha_r over the sequence, the regression family
// solves the unrolled system
//   r_t = y_t - sum_{s<t} e^{Gamma_{t-1}-Gamma_s} eta_s (x_t . x_s) r_s,
//   o_t = sum_{s<=t} e^{Gamma_t-Gamma_s} eta_s (q_t . x_s) r_s
// (inner product: r = y), and the final state is
//   S_L = sum_s e^{Gamma_L-Gamma_s} eta_s r_s x_s^T.
// No state is formed on the way: the kernel walks row blocks I of 64 tokens
// in causal order and, for every earlier column block J, forms the pairwise
// tiles [X_I; Q_I] X_J^T on the tensor core and applies them to the solved
// residuals of block J:
//   [R_I; O_I] -= / += gamma_IJ [X_I X_J^T; Q_I X_J^T] E~_J,
// with E~_J = diag(e^{Gamma_Jend-Gamma_s} eta_s) r_J (kept, bf16, per block)
// and gamma_IJ = e^{Gamma_{I0-1}-Gamma_Jend}.  The decay of a pair splits at
// the block boundaries into a row factor e^{Gamma_{t-1}-Gamma_{I0-1}} (or
// e^{Gamma_t-...}), gamma_IJ and the column factor, each <= 1.  The diagonal
// block then solves its own triangle: R_I = Y_I - D_a (accumulated), E_I =
// (I + M_II)^{-1} R_I, O_I = D_c (accumulated) + (P o Dm)_II E_I.
//
// Windows (Falcon-3/3A, B_w samples per update): token t's unknowns are the
// residuals r_{t,i} of the samples i in its window W_t, and the sums above run
// over the window's samples as well.  A row block then holds 65 - B_w tokens,
// so that the samples their windows reach fill the same 64 rows; the pair
// products apply, per sample row, each earlier block's residual sums
//   R~_J[i] = sum_{s in J, i in W_s} e^{Gamma_Jend-Gamma_s} eta_s r_{s,i},
// and the diagonal block walks its C*B_w system token by token with the
// decayed running sums R <- alpha_t R + eta_t r_t (every factor <= 1):
//   r_{t,i} = y_i - a_t V[i] - (A_II R)[i],  o_t = c_t (accumulated) + P_II[t] R,
// and R after its last token is the block's R~.
//
// One block per (b, h): eight compute warps and an issuing warp.  The pair
// products run on tcgen05 (bf16 operands in
// 128-byte-swizzled shared memory, fp32 accumulators in tensor memory): P1 =
// [X_I; Q_I] X_J^T into one of two accumulators while the previous pair's
// P1 is scaled and rounded into the operand of P2 = [gA; gP] E~_J, which
// accumulates [R; O] over J.  X_J and E~_J come back from the workspace by
// bulk copies, each through a ring of four slots.  The diagonal block works on the
// CUDA cores and the TF32 warp MMAs: T = (I + M_II)^{-1} from its 16 x 16
// diagonal blocks (D) and K = D M_o, T = (I - K + K^2 - K^3) D.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"
#include "warp_tf32.cuh"

namespace falcon {

namespace {

constexpr int BM = 64;         // tokens per block; d_k = d_v = 64
constexpr int NTHC = 256;              // eight compute warps
constexpr int NTHM = NTHC + 32;        // and one warp whose lane 0 issues the products and copies
constexpr int LDM = 72;        // fp32 row stride of the CUDA-core tiles
constexpr int TFM = BM * LDM;  // floats per fp32 tile
constexpr uint32_t TB = 8192;  // one bf16 64 x 64 tile (128-byte rows, 128-byte swizzle)
constexpr int NRING = 4;       // slots of each operand ring
constexpr int NGMAX = 1024;    // row blocks per sequence (L <= 65536)
constexpr uint64_t kWaitNsM = 2000000000ull;  // bounded waits: two seconds

// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t M_AQ = 0;                           // [X_I; Q_I] bf16: A of P1; rows 0-63 also B of the diagonal
constexpr uint32_t M_RING = 2 * TB;                    // NRING slots of X_J bf16 (B of P1) ...
constexpr uint32_t M_ERING = M_RING + NRING * TB;      // ... and NRING slots of E~_J^T bf16 (B of P2)
constexpr uint32_t M_AOP = M_ERING + NRING * TB;       // two [gA; gP] bf16 operands of P2
constexpr uint32_t M_LOOPEND = M_AOP + 2 * 2 * TB;
constexpr uint32_t M_XF = M_LOOPEND;                   // fp32: X_I
constexpr uint32_t M_YF = M_XF + TFM * 4;              // fp32: Y_I, then R_I, then E_I
constexpr uint32_t M_MT = M_YF + TFM * 4;              // fp32: M_II (with the steps)
constexpr uint32_t M_PD = M_MT + TFM * 4;              // fp32: (P o Dm)_II (with the steps)
constexpr uint32_t M_OF = M_PD + TFM * 4;              // fp32: D_c (accumulated O)
constexpr uint32_t M_ET = M_OF + TFM * 4;              // bf16: E~_I^T, staged for the workspace
constexpr uint32_t M_VEC = M_ET + TB;                  // per-token vectors
constexpr uint32_t M_GAM = M_VEC + 9 * BM * 4;        // gamma_IJ of the row block, J < I
constexpr uint32_t M_BAR = M_GAM + NGMAX * 4;
constexpr uint32_t M_SMEM = M_BAR + 192 + 1024;        // + alignment slack
// the inverse's fp32 tiles D, K, K^2, T over the loop region (idle in the diagonal step)
static_assert(4 * TFM * 4 <= M_LOOPEND - M_RING, "inverse scratch must fit over the pair buffers");
static_assert(M_SMEM <= 227 * 1024, "shared memory of one block");
// tensor memory: P1 accumulators at columns 0 and 64, [R; O] at 128
constexpr uint32_t TM_COLS = 256, TM_P1 = 0, TM_ACC = 128;

__device__ unsigned int g_masked_wait_timeouts;

#ifdef FALCON_TC_DEBUG
// block 0, threads 0 (compute) and 256 (the issuer): SM cycles per phase summed over the row blocks
__device__ long long *g_masked_tim;
#define MT_INIT()                    \
    long long mt_acc_[16] = {0};     \
    long long mt_prev_ = clock64();  \
    const bool mt_on_ = blockIdx.x == 0 && (threadIdx.x == 0 || threadIdx.x == 256)
#define MT(k)                                    \
    do {                                         \
        if (mt_on_) {                            \
            const long long n_ = clock64();      \
            mt_acc_[k] += n_ - mt_prev_;         \
            mt_prev_ = n_;                       \
        }                                        \
    } while (0)
#define MT_END()                                                                                    \
    do {                                                                                            \
        if (mt_on_ && g_masked_tim)                                                                 \
            for (int i_ = 0; i_ < 16; ++i_) g_masked_tim[(threadIdx.x ? 16 : 0) + i_] = mt_acc_[i_]; \
    } while (0)
#else
#define MT_INIT()
#define MT(k)
#define MT_END()
#endif

// every product here: M = 128, N = 64, K = 64, both operands K-major
constexpr uint32_t kIdesc = tc::idesc_bf16(128, 64, 0, 0);
// descriptor units (16 bytes) of one bf16 tile
constexpr uint32_t kTileDesc = TB >> 4;

// barrier `id` over the first n threads of the block; true when pred holds on all of them
__device__ __forceinline__ bool named_sync_and(uint32_t id, uint32_t n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <bool TA, bool TB, bool SK = false>
__device__ __forceinline__ void mma64(const float *A, const float *B, float (&acc)[4][4], int kb, int ke,
                                      const float *sk = nullptr) {
    wt::mma64<LDM, TA, TB, SK>(A, B, acc, kb, ke, sk);
}

}  // namespace

template <int W>
__global__ void __launch_bounds__(NTHM, 1)
    masked_tc_kernel(FwdParams p, uint8_t *xs_ws, uint8_t *es_ws, float *gend_ws) {
    // tokens per row block: its samples (the window reaches W - 1 back) fill the 64 rows
    constexpr int TOK = BM + 1 - W;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = tc::smem_u32(smem_raw);
    uint8_t *sm = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sb = tc::smem_u32(sm);
    float *XF = reinterpret_cast<float *>(sm + M_XF), *YF = reinterpret_cast<float *>(sm + M_YF);
    float *MT = reinterpret_cast<float *>(sm + M_MT), *PD = reinterpret_cast<float *>(sm + M_PD);
    float *OF = reinterpret_cast<float *>(sm + M_OF);
    float *DI = reinterpret_cast<float *>(sm + M_RING), *KI = DI + TFM, *K2 = KI + TFM, *TI = K2 + TFM;
    float *vec = reinterpret_cast<float *>(sm + M_VEC);
    float *vG = vec, *veta = vec + BM, *vla = vec + 2 * BM, *va = vec + 3 * BM, *vc = vec + 4 * BM,
          *vb = vec + 5 * BM, *vsq = vec + 6 * BM, *vbeta = vec + 7 * BM, *valpha = vec + 8 * BM;
    // window system (W > 1): the sample Gram, the token-sample scores, the
    // accumulated pair terms per sample row and the block's residual sums
    float *AT = MT, *PT = PD, *VT = DI, *RT = KI;
    float *vgam = reinterpret_cast<float *>(sm + M_GAM);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + M_BAR);
    uint64_t *txb = bar, *teb = bar + NRING, *bp1 = bar + 2 * NRING, *bp2 = bp1 + 2, *bd = bp2 + 2, *bao = bd + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bao + 2);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool compute = tid < NTHC, issuer = tid == NTHC;  // warps 0-7 compute; warp 8 lane 0 issues
    const int quarter = warp & 3, chalf = warp >> 2;
    const int row = quarter * 32 + lane;  // tensor-memory lane of a compute thread
    const bool reg = p.variant == F1 || p.variant == F3;
    const int L = p.L, nb = (L + TOK - 1) / TOK;
    const size_t bh = blockIdx.x;
    const float lam = p.lambda[bh % p.H];
    const __nv_bfloat16 *kh = static_cast<const __nv_bfloat16 *>(p.k) + bh * (size_t)L * BM;
    const __nv_bfloat16 *qh = static_cast<const __nv_bfloat16 *>(p.q) + bh * (size_t)L * BM;
    const __nv_bfloat16 *vh = static_cast<const __nv_bfloat16 *>(p.v) + bh * (size_t)L * BM;
    const __nv_bfloat16 *bth = static_cast<const __nv_bfloat16 *>(p.beta) + bh * (size_t)L;
    __nv_bfloat16 *oh = static_cast<__nv_bfloat16 *>(p.out) + bh * (size_t)L * BM;
    uint8_t *xs = xs_ws + bh * (size_t)nb * TB;
    uint8_t *es = es_ws + bh * (size_t)nb * TB;
    float *gend = gend_ws + bh * (size_t)nb;

    if (issuer) {
        for (int i = 0; i < 2 * NRING + 5; ++i) tc::mbar_init(&bar[i], 1);
        tc::mbar_init(&bao[0], NTHC);
        tc::mbar_init(&bao[1], NTHC);
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tlane = tbase + ((uint32_t)(quarter * 32) << 16);

    // completion counts.  The compute threads count the product barriers
    // (P1, P2, the diagonal product); the issuer counts the operand
    // hand-offs, the P2 issued per accumulator and the ring loads.
    uint32_t n1[2] = {0u, 0u}, n2[2] = {0u, 0u}, ndg = 0u;
    uint32_t na[2] = {0u, 0u}, i2[2] = {0u, 0u};
    uint32_t lx[NRING] = {0u, 0u, 0u, 0u}, cx[NRING] = {0u, 0u, 0u, 0u};
    uint32_t le[NRING] = {0u, 0u, 0u, 0u}, ce[NRING] = {0u, 0u, 0u, 0u};
    bool ok = true;
    float Gprev = 0.f;  // Gamma_{I0-1}
    float sacc[4][4];   // S (this compute warp's 16 x 32 block), relative to the last block's end
    wt::zero(sacc);
    MT_INIT();

    // issuer: X_J into its ring slot, E~_J^T into its own; the waits for them
    auto load_x = [&](int J) {
        const int s = J % NRING;
        tc::mbar_arrive_expect_tx(&txb[s], TB);
        tc::bulk_load(sb + M_RING + (uint32_t)s * TB, xs + (size_t)J * TB, TB, &txb[s]);
        ++lx[s];
    };
    auto load_e = [&](int J) {
        const int s = J % NRING;
        tc::mbar_arrive_expect_tx(&teb[s], TB);
        tc::bulk_load(sb + M_ERING + (uint32_t)s * TB, es + (size_t)J * TB, TB, &teb[s]);
        ++le[s];
    };
    auto wait_x = [&](int J) {
        const int s = J % NRING;
        const bool r = tc::mbar_wait_timeout(&txb[s], cx[s] & 1u, kWaitNsM);
        ++cx[s];
        return r;
    };
    auto wait_e = [&](int J) {
        const int s = J % NRING;
        const bool r = tc::mbar_wait_timeout(&teb[s], ce[s] & 1u, kWaitNsM);
        ++ce[s];
        return r;
    };
    // the operand descriptors, built once
    const uint64_t dAQ = tc::sdesc_sw128(sb + M_AQ, 16, 1024);
    const uint64_t dX0 = tc::sdesc_sw128(sb + M_RING, 16, 1024);
    const uint64_t dE0 = tc::sdesc_sw128(sb + M_ERING, 16, 1024);
    const uint64_t dA0 = tc::sdesc_sw128(sb + M_AOP, 16, 1024);
    auto issue_p1 = [&](int J) {  // P1(J) = [X_I; Q_I] X_J^T into accumulator J & 1
        tc::mma_k64(tbase + TM_P1 + (uint32_t)(J & 1) * 64, dAQ, dX0 + (uint64_t)(J % NRING) * kTileDesc, kIdesc,
                    false);
        tc::mma_commit(&bp1[J & 1]);
    };

    for (int I = 0; I < nb; ++I) {
        const int I0 = I * TOK, n = min(TOK, L - I0);
        // sample row r holds sample i0 + r (the window of token I0 + tau covers
        // rows tau .. tau + W - 1); rows from nsr on, and samples before the
        // sequence, are empty
        const int i0 = I0 - (W - 1), nsr = n + W - 1;
        // ---- the block's inputs: samples x_i = phi(k_{i-1}) (prefix pair;
        //      phi(k_i) same-step) with their targets y_i = v_i, q, the window
        //      energies, the steps and the decays
        if (issuer) tc::bulk_wait_read();  // the stores of the last block have read AQ and ET
        __syncthreads();
        if (compute) {
            uint4 lq[2], lv[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int e = tid + NTHC * j, r = e >> 3, c = e & 7;  // 16-byte piece: row r, columns 8c..
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                lq[j] = r < n ? wt::ld16(qh + (size_t)(I0 + r) * BM + 8 * c) : z;
                lv[j] = (r < nsr && i0 + r >= 0) ? wt::ld16(vh + (size_t)(i0 + r) * BM + 8 * c) : z;
            }
            uint32_t kw[8];
            float bv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = warp * 8 + i, si = i0 + r, kr = p.pairing == 0 ? si - 1 : si;
                kw[i] = (r < nsr && si >= 0 && kr >= 0)
                            ? *reinterpret_cast<const uint32_t *>(kh + (size_t)kr * BM + 2 * lane) : 0u;
                bv[i] = r < n ? __bfloat162float(bth[I0 + r]) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = warp * 8 + i;
                const float x0 = __uint_as_float(kw[i] << 16), x1 = __uint_as_float(kw[i] & 0xffff0000u);
                const float ss = group_sum<32>(x0 * x0 + x1 * x1);
                const float inv = p.phi != 0 ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
                const float y0 = x0 * inv, y1 = x1 * inv;
                *reinterpret_cast<float2 *>(XF + r * LDM + 2 * lane) = make_float2(y0, y1);
                *reinterpret_cast<uint32_t *>(sm + M_AQ + tc::sw128(r, lane >> 2) + (lane & 3) * 4) = pack2(y0, y1);
                if (lane == 0) {
                    vsq[r] = ss * inv * inv;  // the sample's energy (0: no sample)
                    vbeta[r] = bv[i];
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int e = tid + NTHC * j, r = e >> 3, c = e & 7;
                *reinterpret_cast<uint4 *>(sm + M_AQ + tc::sw128(64 + r, c)) = lq[j];
                wt::st8(YF + r * LDM + 8 * c, lv[j]);
            }
            tc::named_sync(1, NTHC);
            if (tid < BM) {  // token tau: its window's energy, step and decay
                const int t = tid;
                float nn = 0.f;
#pragma unroll
                for (int m = 0; m < W; ++m) nn += vsq[min(t + m, BM - 1)];
                float eta = 0.f, alpha = 1.f;
                if (t < n) step_and_decay(vbeta[t], nn, p.eps, lam, eta, alpha);
                veta[t] = eta;
                valpha[t] = alpha;
                vla[t] = __logf(alpha);
            }
            tc::named_sync(1, NTHC);
            if (warp == 0) {  // block-local cumulative log decay G_t
                float la[2] = {vla[lane], vla[lane + 32]};
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
            tc::named_sync(1, NTHC);
            const float GE = vG[BM - 1];
            if (tid < BM) {
                const int t = tid;
                va[t] = __expf(t > 0 ? vG[t - 1] : 0.f);   // e^{Gamma_{t-1} - Gamma_{I0-1}}
                vc[t] = __expf(vG[t]);                      // e^{Gamma_t - Gamma_{I0-1}}
                vb[t] = __expf(GE - vG[t]) * veta[t];       // e^{Gamma_Iend - Gamma_t} eta_t
                vla[t] = __expf(-vG[t]) * veta[t];          // e^{Gamma_{I0-1} - Gamma_t} eta_t (the logs are read)
            }
            if (tid == 0) gend[I] = Gprev + GE;
            tc::fence_proxy_async();
        }
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        const float GE = vG[BM - 1];
        const bool fact = GE > -80.f;  // every e^{-G_t} of the block inside the fp32 range
        if (issuer) {  // X_I for the later row blocks
            tc::bulk_store(xs + (size_t)I * TB, sb + M_AQ, TB);
            tc::bulk_commit();
        }
        MT(0);

        // ---- the pairs (I, J < I).  The compute warps turn P1(J) into the
        //      operand [gA; gP] of P2(J) and hand it over through an mbarrier;
        //      the issuer runs P2(J) and P1 two pairs ahead, and keeps X_J
        //      four pairs and E~_J three pairs ahead in their rings
        if (I > 0) {
            if (issuer) {
                // every earlier X_J and E~_J has landed in the workspace (the
                // store of X_I, the newest group, may still be in flight)
                asm volatile("cp.async.bulk.wait_group 1;" ::: "memory");
                for (int J = 0; J < min(NRING, I); ++J) load_x(J);
                for (int J = 0; J < min(NRING - 1, I); ++J) load_e(J);
                bool r = wait_x(0);
                if (r) issue_p1(0);
                if (r && I > 1) {
                    r = wait_x(1);
                    if (r) issue_p1(1);
                }
                ok = r;
            } else if (compute) {
                for (int J = tid; J < I; J += NTHC) vgam[J] = __expf(Gprev - gend[J]);
            }
            ok = __syncthreads_and(ok);
            MT(1);
            if (compute) {
                for (int J = 0; J < I && ok; ++J) {
                    const int b = J & 1;
                    // P1(J) -> this thread's 32 columns of its lane
                    bool w = tc::mbar_wait_timeout(&bp1[b], n1[b] & 1u, kWaitNsM);
                    ++n1[b];
                    __syncwarp();
                    tc::fence_after_sync();
                    float v[32];
                    tc::tmem_ld32(tlane + TM_P1 + b * 64 + chalf * 32, v);
                    tc::tmem_wait_ld();
                    MT(2);
                    // [gA; gP] of this pair into operand b once P2(J-2) has read it
                    const float g = vgam[J];
                    if (J >= 2) {
                        w = tc::mbar_wait_timeout(&bp2[b], n2[b] & 1u, kWaitNsM) && w;
                        ++n2[b];
                    }
                    const uint32_t aop = M_AOP + (uint32_t)b * 2 * TB;
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint4 u;
                        u.x = pack2(g * v[c4 * 8 + 0], g * v[c4 * 8 + 1]);
                        u.y = pack2(g * v[c4 * 8 + 2], g * v[c4 * 8 + 3]);
                        u.z = pack2(g * v[c4 * 8 + 4], g * v[c4 * 8 + 5]);
                        u.w = pack2(g * v[c4 * 8 + 6], g * v[c4 * 8 + 7]);
                        *reinterpret_cast<uint4 *>(sm + aop + tc::sw128(row, chalf * 4 + c4)) = u;
                    }
                    tc::fence_proxy_async();
                    tc::fence_before_sync();
                    // accumulator b is read and operand b written: hand both over
                    tc::mbar_arrive(&bao[b]);
                    ok = w;
                    MT(3);
                }
                if (ok) {
                    // the last two P2 (the others have been counted)
                    for (int J = max(0, I - 2); J < I && ok; ++J) {
                        const int b = J & 1;
                        ok = tc::mbar_wait_timeout(&bp2[b], n2[b] & 1u, kWaitNsM);
                        ++n2[b];
                    }
                }
            } else if (issuer) {
                for (int J = 0; J < I && ok; ++J) {
                    const int b = J & 1;
                    bool r = tc::mbar_wait_timeout(&bao[b], na[b] & 1u, kWaitNsM);
                    ++na[b];
                    tc::fence_after_sync();
                    MT(4);
                    // P2(J): [R; O] += [gA; gP] E~_J
                    r = r && wait_e(J);
                    MT(12);
                    if (r) {
                        tc::mma_k64(tbase + TM_ACC, dA0 + (uint64_t)b * 2 * kTileDesc,
                                    dE0 + (uint64_t)(J % NRING) * kTileDesc, kIdesc, J > 0);
                        tc::mma_commit(&bp2[b]);
                        ++i2[b];
                    }
                    MT(10);
                    // P1(J+2) into accumulator b, read out by every compute thread
                    if (r && J + 2 < I) {
                        r = wait_x(J + 2);
                        if (r) issue_p1(J + 2);
                    }
                    MT(11);
                    // X_{J+4} into the slot of X_J (P1(J) is done)
                    if (r && J + NRING < I) load_x(J + NRING);
                    // E~_{J+3} into the slot of E~_{J-1} once P2(J-1), the newest
                    // product of accumulator b ^ 1, is done
                    if (r && J + NRING - 1 < I) {
                        if (J >= 1) r = tc::mbar_wait_timeout(&bp2[b ^ 1], (i2[b ^ 1] - 1u) & 1u, kWaitNsM);
                        if (r) load_e(J + NRING - 1);
                    }
                    MT(5);
                    if (!r) ok = false;
                }
            }
            ok = __syncthreads_and(ok);
            if (!ok) break;
            MT(6);
        }

        // ---- the diagonal block: [A_II; P_II] = [X_I; Q_I] X_I^T
        if (issuer) {
            tc::mma_k64(tbase + TM_P1, dAQ, dAQ, kIdesc, false);
            tc::mma_commit(bd);
        }
        if (compute) {
            {
                const bool w = tc::mbar_wait_timeout(bd, ndg & 1u, kWaitNsM);
                ++ndg;
                __syncwarp();
                tc::fence_after_sync();
                ok = w;
            }
            float v[32], r[32];
            tc::tmem_ld32(tlane + TM_P1 + chalf * 32, v);
            if (I > 0) tc::tmem_ld32(tlane + TM_ACC + chalf * 32, r);
            tc::tmem_wait_ld();
            if (I == 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = 0.f;
            }
            if (W > 1) {
                // window system: the sample Gram and V (rows 0-63, regression),
                // the token-sample scores and D_c (accumulated O) (rows 64-127)
                if (quarter < 2) {
                    if (reg) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            AT[row * LDM + chalf * 32 + i] = v[i];
                            VT[row * LDM + chalf * 32 + i] = r[i];
                        }
                    }
                } else {
                    const int t = row - 64;
                    const float c = vc[t];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        PT[t * LDM + chalf * 32 + i] = v[i];
                        OF[t * LDM + chalf * 32 + i] = c * r[i];
                    }
                }
            } else if (quarter < 2) {  // rows 0-63 (regression): M_II (with the steps), R = Y - D_a (accumulated)
                if (reg) {
                    const int t = row;
                    const float gm = t > 0 ? vG[t - 1] : 0.f, a = va[t];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int s2 = chalf * 32 + i;
                        // e^{G_{t-1} - G_s} eta_s: factorised while the block's G stays above -80
                        const float f = fact ? a * vla[s2] : __expf(gm - vG[s2]) * veta[s2];
                        MT[t * LDM + s2] = s2 < t ? f * v[i] : 0.f;
                        YF[t * LDM + s2] -= a * r[i];
                    }
                }
            } else {  // rows 64-127: (P o Dm)_II (with the steps) and D_c (accumulated)
                const int t = row - 64;
                const float gt = vG[t], c = vc[t];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int s2 = chalf * 32 + i;
                    const float f = fact ? c * vla[s2] : __expf(gt - vG[s2]) * veta[s2];
                    PD[t * LDM + s2] = s2 <= t ? f * v[i] : 0.f;
                    OF[t * LDM + s2] = c * r[i];
                }
            }
            tc::fence_before_sync();
            ok = named_sync_and(1, NTHC, ok);
        }
        MT(7);
        if (compute && ok && W == 1) {
            const int rb = (warp & 3) * 16, cb = (warp >> 2) * 32;
            float acc[4][4];
            if (reg) {
                // ---- T = (I + M_II)^{-1}: D, the diagonal 16 x 16 blocks' inverses
                //      (one column of a block per thread, threads 0-63); zeros elsewhere
                if (tid < 64) {
                    const int o = (tid >> 4) * 16, j = tid & 15;
                    float col[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float sv = i == j ? 1.f : 0.f;
#pragma unroll
                        for (int s2 = 0; s2 < i; ++s2) sv -= MT[(o + i) * LDM + o + s2] * col[s2];
                        col[i] = sv;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) DI[(o + i) * LDM + o + j] = col[i];
                } else {
                    for (int e = tid - 64; e < BM * BM; e += NTHC - 64) {
                        const int r2 = e >> 6, s2 = e & 63;
                        if ((r2 >> 4) != (s2 >> 4)) DI[r2 * LDM + s2] = 0.f;
                    }
                }
                tc::named_sync(1, NTHC);
                // K = D M_o: D M on the blocks below the diagonal (D reads its own block only)
                wt::zero(acc);
                mma64<false, false>(DI, MT, acc, rb, rb + 16);
                wt::each(acc, [&](int r2, int s2, float &val) { KI[r2 * LDM + s2] = (s2 >> 4) < (r2 >> 4) ? val : 0.f; });
                tc::named_sync(1, NTHC);
                wt::zero(acc);
                if (rb > 0) mma64<false, false>(KI, KI, acc, 0, rb);
                wt::each(acc, [&](int r2, int s2, float &val) { K2[r2 * LDM + s2] = val; });
                tc::named_sync(1, NTHC);
                wt::zero(acc);
                if (rb > 0) mma64<false, false>(KI, K2, acc, 0, rb);
                wt::each(acc, [&](int r2, int s2, float &val) {
                    TI[r2 * LDM + s2] = (r2 == s2 ? 1.f : 0.f) - KI[r2 * LDM + s2] + K2[r2 * LDM + s2] - val;
                });
                tc::named_sync(1, NTHC);
                // T = (I - K + K^2 - K^3) D: each warp reads only the block of the sum it writes
                wt::zero(acc);
                {
                    const int ke = min(cb + 32, rb + 16);
                    if (ke > cb) mma64<false, false>(TI, DI, acc, cb, ke);
                }
                __syncwarp();
                wt::each(acc, [&](int r2, int s2, float &val) { TI[r2 * LDM + s2] = val; });
                tc::named_sync(1, NTHC);
                // E = T R (T lower: k <= r)
                wt::zero(acc);
                mma64<false, false>(TI, YF, acc, 0, rb + 16);
                tc::named_sync(1, NTHC);
                wt::each(acc, [&](int r2, int j, float &val) { YF[r2 * LDM + j] = val; });
                tc::named_sync(1, NTHC);
            }
            MT(8);
            // ---- O_I = D_c (accumulated) + (P o Dm)_II E_I
            wt::zero(acc);
            mma64<false, false>(PD, YF, acc, 0, rb + 16);
            {
                const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int r2 = rb + g + 8 * h2, j = cb + nt * 8 + 2 * t4;
                        if (r2 < n) {
                            const float o0 = acc[nt][2 * h2] + OF[r2 * LDM + j];
                            const float o1 = acc[nt][2 * h2 + 1] + OF[r2 * LDM + j + 1];
                            *reinterpret_cast<uint32_t *>(oh + (size_t)(I0 + r2) * BM + j) = pack2(o0, o1);
                        }
                    }
            }
            // ---- E~_I^T (bf16, swizzled: row j holds b_s E[s][j] over s) for the later
            //      row blocks, and S <- e^{G_Iend} S + E~_I^T X_I
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int e = tid + NTHC * k2, j = e >> 3, c = e & 7;
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = vb[8 * c + i] * YF[(8 * c + i) * LDM + j];
                uint4 u;
                u.x = pack2(f[0], f[1]);
                u.y = pack2(f[2], f[3]);
                u.z = pack2(f[4], f[5]);
                u.w = pack2(f[6], f[7]);
                *reinterpret_cast<uint4 *>(sm + M_ET + tc::sw128(j, c)) = u;
            }
            const float gI = __expf(GE);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[nt][e] *= gI;
            mma64<true, false, true>(YF, XF, sacc, 0, 64, vb);
            tc::fence_proxy_async();
        }
        if (compute && ok && W > 1) {
            // ---- the window system in token order.  Thread (j, q): value
            //      channel j, sample rows 16q..16q+15 of the running sums
            //        R[r] = sum_{s <= t} e^{G_t - G_s} eta_s r_{s, r}   (r in W_s),
            //      R <- alpha_t R + eta_t r_t after token t.  Token t's residuals
            //        r_{t, rho} = y_rho - a_t V[rho] - (A R)[rho], rho = t .. t+W-1
            //      (inner product: r = y), and o_t = D_c (accumulated) + P[t] R.
            //      After the last token R is the block's residual sum per sample
            //      row, weighted to the block's end.
            const int jc = tid >> 2, qr = tid & 3;
            float racc[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) racc[q] = 0.f;
            // tokens in groups of 16 (t = 16 g + v, v unrolled): token t's rows
            // t + m fall in this thread's rows 16 qr .. 16 qr + 15 at the fixed
            // index v + m when qr == g, or v + m - 16 when qr == g + 1
            for (int g = 0; 16 * g < n; ++g) {
#pragma unroll
                for (int v = 0; v < 16; ++v) {
                    const int t = 16 * g + v;
                    if (t >= n) break;
                    const float a = va[t], eta = veta[t], alpha = valpha[t];
                    float rm[W];
#pragma unroll
                    for (int m = 0; m < W; ++m) {
                        const int rho = t + m;
                        float res = YF[rho * LDM + jc];
                        if (reg) {
                            const float4 *ar = reinterpret_cast<const float4 *>(AT + rho * LDM + 16 * qr);
                            float d0 = 0.f, d1 = 0.f;
#pragma unroll
                            for (int q4 = 0; q4 < 4; q4 += 2) {
                                const float4 av = ar[q4], aw = ar[q4 + 1];
                                d0 += av.x * racc[4 * q4] + av.y * racc[4 * q4 + 1] + av.z * racc[4 * q4 + 2] +
                                      av.w * racc[4 * q4 + 3];
                                d1 += aw.x * racc[4 * q4 + 4] + aw.y * racc[4 * q4 + 5] +
                                      aw.z * racc[4 * q4 + 6] + aw.w * racc[4 * q4 + 7];
                            }
                            float d = d0 + d1;
                            d += __shfl_xor_sync(0xffffffffu, d, 1);
                            d += __shfl_xor_sync(0xffffffffu, d, 2);
                            res -= a * VT[rho * LDM + jc] + d;
                        }
                        rm[m] = eta * res;
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q) racc[q] *= alpha;
#pragma unroll
                    for (int m = 0; m < W; ++m) {
                        if (v + m < 16) {
                            if (qr == g) racc[v + m] += rm[m];
                        } else {
                            if (qr == g + 1) racc[v + m - 16] += rm[m];
                        }
                    }
                    const float4 *pr = reinterpret_cast<const float4 *>(PT + t * LDM + 16 * qr);
                    float o0 = 0.f, o1 = 0.f;
#pragma unroll
                    for (int q4 = 0; q4 < 4; q4 += 2) {
                        const float4 pv = pr[q4], pw = pr[q4 + 1];
                        o0 += pv.x * racc[4 * q4] + pv.y * racc[4 * q4 + 1] + pv.z * racc[4 * q4 + 2] +
                              pv.w * racc[4 * q4 + 3];
                        o1 += pw.x * racc[4 * q4 + 4] + pw.y * racc[4 * q4 + 5] + pw.z * racc[4 * q4 + 6] +
                              pw.w * racc[4 * q4 + 7];
                    }
                    float o = o0 + o1;
                    o += __shfl_xor_sync(0xffffffffu, o, 1);
                    o += __shfl_xor_sync(0xffffffffu, o, 2);
                    if (qr == 0) oh[(size_t)(I0 + t) * BM + jc] = __float2bfloat16_rn(OF[t * LDM + jc] + o);
                }
            }
            // the block's residual sums: fp32 for the state, bf16 (row j, sample
            // rows along K) for the later row blocks
#pragma unroll
            for (int q = 0; q < 16; ++q) RT[(16 * qr + q) * LDM + jc] = racc[q];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                uint4 u;
                u.x = pack2(racc[8 * h2 + 0], racc[8 * h2 + 1]);
                u.y = pack2(racc[8 * h2 + 2], racc[8 * h2 + 3]);
                u.z = pack2(racc[8 * h2 + 4], racc[8 * h2 + 5]);
                u.w = pack2(racc[8 * h2 + 6], racc[8 * h2 + 7]);
                *reinterpret_cast<uint4 *>(sm + M_ET + tc::sw128(jc, 2 * qr + h2)) = u;
            }
            tc::named_sync(1, NTHC);
            // S <- e^{G_Iend} S + R^T X
            const float gI = __expf(GE);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[nt][e] *= gI;
            mma64<true, false>(RT, XF, sacc, 0, 64);
            tc::fence_proxy_async();
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(ok);
        if (!ok) break;
        if (issuer) {
            tc::bulk_store(es + (size_t)I * TB, sb + M_ET, TB);
            tc::bulk_commit();
        }
        Gprev += GE;
        MT(9);
    }

    MT_END();
    if (p.final_state && ok && compute)
        wt::each(sacc, [&](int j, int i, float &val) { p.final_state[(bh * BM + j) * BM + i] = val; });
    if (issuer) {
        tc::bulk_wait_all();
        if (!ok) {
            atomicAdd(&g_masked_wait_timeouts, 1u);
            // loads still in flight must land before the block leaves
            for (int s2 = 0; s2 < NRING; ++s2) {
                if (lx[s2] > cx[s2]) (void)tc::mbar_wait_timeout(&txb[s2], (lx[s2] - 1u) & 1u, kWaitNsM);
                if (le[s2] > ce[s2]) (void)tc::mbar_wait_timeout(&teb[s2], (le[s2] - 1u) & 1u, kWaitNsM);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, TM_COLS);
}

// ------------------------------------------------------------ launcher
namespace {

size_t al256m(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

bool al16m(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// samples per update the kernel runs with: 1 (Falcon-1/1A, or a window of
// one), 2-4 (Falcon-3/3A); 0: not covered
int masked_tc_window(const FwdParams &p) {
    if (p.dk != BM || p.dv != BM || p.form != 1 || p.L <= 0) return 0;
    int w = 0;
    if (p.variant == F1 || p.variant == F1A) w = 1;
    if ((p.variant == F3 || p.variant == F3A) && p.window >= 1 && p.window <= 4) w = p.window;
    if (w == 0) return 0;
    const int tok = BM + 1 - w;
    return (p.L + tok - 1) / tok <= NGMAX ? w : 0;
}

bool masked_tc_covers(const FwdParams &p) { return masked_tc_window(p) != 0; }

size_t masked_tc_ws_bytes(const FwdParams &p) {
    const int w = masked_tc_window(p);
    const size_t BH = (size_t)p.B * p.H, nb = (p.L + BM - w) / (BM + 1 - (w ? w : 1));
    return 2 * al256m(BH * nb * TB) + al256m(BH * nb * sizeof(float));
}

namespace {

template <int W>
int launch_w(const FwdParams &p, void *ws, cudaStream_t s) {
    constexpr int TOK = BM + 1 - W;
    const size_t BH = (size_t)p.B * p.H, nb = (p.L + TOK - 1) / TOK;
    uint8_t *base = static_cast<uint8_t *>(ws);
    uint8_t *xs = base, *es = base + al256m(BH * nb * TB);
    float *gend = reinterpret_cast<float *>(es + al256m(BH * nb * TB));
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr[dev]) {
        cudaFuncSetAttribute(masked_tc_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)M_SMEM);
        if (dev >= 0 && dev < 64) attr[dev] = true;
    }
    masked_tc_kernel<W><<<(unsigned)BH, NTHM, M_SMEM, s>>>(p, xs, es, gend);
    return cudaGetLastError() == cudaSuccess ? 0 : -7;
}

}  // namespace

// 1: not covered (the caller takes the CUDA-core path); 0 launched; < 0 an error
int launch_masked_tc(const FwdParams &p, void *ws, cudaStream_t s) {
    const int w = masked_tc_window(p);
    if (w == 0) return 1;
    if (!al16m(p.q) || !al16m(p.k) || !al16m(p.v) || !al16m(p.out)) return 1;
    switch (w) {
        case 1: return launch_w<1>(p, ws, s);
        case 2: return launch_w<2>(p, ws, s);
        case 3: return launch_w<3>(p, ws, s);
        default: return launch_w<4>(p, ws, s);
    }
}

#ifdef FALCON_TC_DEBUG
extern "C" int falcon_masked_debug_timer_set(long long *ptr) {
    return cudaMemcpyToSymbol(g_masked_tim, &ptr, sizeof(ptr)) == cudaSuccess ? 0 : -1;
}
#endif

unsigned int masked_wait_timeouts() {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_masked_wait_timeouts, sizeof(v));
    return v;
}

}  // namespace falcon
