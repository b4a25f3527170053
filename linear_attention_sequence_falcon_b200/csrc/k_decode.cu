// k_decode.cu -- one recurrent step per sequence (decode) and the decode carry
// after a prefill ("recurrent: O(d^2) per step, for inference", page "Fast
// Weight Attention：用于持续学习的快速权重注意力", 核心方法 3).
//
// The step is bound by streaming the fp32 state: every row of S is read once
// and written once.  One thread block owns one (n,h): DK/4 lanes hold a row as
// one float4 each (a 128-wide row is one fully coalesced 512-byte warp
// access), four row passes are loaded before any is used to keep several
// loads in flight per thread, and the two dot products a row needs (S_j.x_m
// for every window sample, S_j.q) are reduced together by xor-shuffles.  The
// read uses o_j = alpha (S_j.q) + eta sum_m e_m (x_m.q), so the updated row
// is never re-read.  Because one block owns the (n,h), the carry (x_prev and
// the window) is updated in place without races.
#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {

template <typename T, int DK>
__global__ void __launch_bounds__(256) decode_kernel(DecodeParams p) {
    constexpr int LPR = DK / 4;
    constexpr int RPW = 32 / LPR;
    constexpr int NW = 8;
    constexpr int RPP = NW * RPW;  // rows per pass
    constexpr int U = 4;           // passes in flight
    __shared__ __align__(16) float xw[kMaxWindow][DK];
    __shared__ float yw[kMaxWindow][128];
    __shared__ __align__(16) float qv[DK];
    __shared__ float kn[DK];
    __shared__ float xq[kMaxWindow];
    __shared__ float sqm[kMaxWindow];
    __shared__ float knorm;

    const VariantInfo vi = variant_info(p.variant, p.window);
    const int w = vi.window;
    const int nh = blockIdx.x;
    const int h = nh % p.H;
    const int dv = p.dv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T *q = static_cast<const T *>(p.q) + (size_t)nh * DK;
    const T *k = static_cast<const T *>(p.k) + (size_t)nh * DK;
    const T *v = static_cast<const T *>(p.v) + (size_t)nh * dv;
    const T *beta = static_cast<const T *>(p.beta) + (size_t)nh * (vi.per_channel ? dv : 1);
    const bool same = p.pairing != 0;  // same-step pair: the current sample is (phi(k_t), v_t)
    float *xp = p.x_prev ? p.x_prev + (size_t)nh * DK : nullptr;
    float *win = p.win ? p.win + (size_t)nh * (w - 1) * (DK + dv) : nullptr;

    // stage the window (oldest first), the current sample (x_prev, v_t), q and k
    for (int i = threadIdx.x; i < DK; i += blockDim.x) {
        xw[w - 1][i] = same ? 0.f : xp[i];
        qv[i] = to_f32(q[i]);
        kn[i] = to_f32(k[i]);
    }
    for (int i = threadIdx.x; i < dv; i += blockDim.x) yw[w - 1][i] = to_f32(v[i]);
    for (int i = threadIdx.x; i < (w - 1) * (DK + dv); i += blockDim.x) {
        const int m = i / (DK + dv), c = i % (DK + dv);
        const float val = win[i];
        if (c < DK) xw[m][c] = val; else yw[m][c - DK] = val;
    }
    __syncthreads();
    if (same) {  // the current sample is phi(k_t): its norm first
        if (warp == 0) {
            float a = 0.f;
            for (int c = lane; c < DK; c += 32) a += kn[c] * kn[c];
            a = group_sum<32>(a);
            if (lane == 0) knorm = a;
        }
        __syncthreads();
        const float inv = knorm > 0.f ? rsqrtf(knorm) : 0.f;
        for (int i = threadIdx.x; i < DK; i += blockDim.x) xw[w - 1][i] = kn[i] * inv;
        __syncthreads();
    }
    if (warp < w) {
        float a = 0.f, b = 0.f;
        for (int c = lane; c < DK; c += 32) {
            a += xw[warp][c] * qv[c];
            b += xw[warp][c] * xw[warp][c];
        }
        a = group_sum<32>(a);
        b = group_sum<32>(b);
        if (lane == 0) { xq[warp] = a; sqm[warp] = b; }
    }
    if (warp == NW - 1) {
        float a = 0.f;
        for (int c = lane; c < DK; c += 32) a += kn[c] * kn[c];
        a = group_sum<32>(a);
        if (lane == 0) knorm = a;
    }
    __syncthreads();
    float n = 0.f;
    for (int m = 0; m < w; ++m) n += sqm[m];
    const float lam = p.lambda[h];
    float eta_s = 0.f, alpha_s = 1.f;
    if (!vi.per_channel) step_and_decay(to_f32(beta[0]), n, p.eps, lam, eta_s, alpha_s);

    const int sl = lane % LPR;
    const int rsub = warp * RPW + lane / LPR;
    float4 xm[kMaxWindow];
#pragma unroll
    for (int m = 0; m < kMaxWindow; ++m)
        if (m < w) xm[m] = *reinterpret_cast<const float4 *>(&xw[m][sl * 4]);
    const float4 q4 = *reinterpret_cast<const float4 *>(&qv[sl * 4]);
    float *S = p.state + (size_t)nh * dv * DK;
    T *out = static_cast<T *>(p.out) + (size_t)nh * dv;

    for (int base = 0; base < dv; base += RPP * U) {
        float4 s4[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int row = base + u * RPP + rsub;
            if (row < dv) s4[u] = *reinterpret_cast<const float4 *>(S + (size_t)row * DK + sl * 4);
            else s4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int row = base + u * RPP + rsub;
            const float4 s = s4[u];
            float sq = s.x * q4.x + s.y * q4.y + s.z * q4.z + s.w * q4.w;
            sq = group_sum<LPR>(sq);
            float e[kMaxWindow];
#pragma unroll
            for (int m = 0; m < kMaxWindow; ++m) {
                e[m] = 0.f;
                if (m < w) {
                    float d = 0.f;
                    if (vi.regression) {
                        d = s.x * xm[m].x + s.y * xm[m].y + s.z * xm[m].z + s.w * xm[m].w;
                        d = group_sum<LPR>(d);
                    }
                    const float y = row < dv ? yw[m][row] : 0.f;
                    e[m] = vi.regression ? y - d : y;
                }
            }
            float eta = eta_s, alpha = alpha_s;
            if (vi.per_channel && row < dv) step_and_decay(to_f32(beta[row]), n, p.eps, lam, eta, alpha);
            float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
            float gq = 0.f;
#pragma unroll
            for (int m = 0; m < kMaxWindow; ++m)
                if (m < w) {
                    g.x += e[m] * xm[m].x; g.y += e[m] * xm[m].y;
                    g.z += e[m] * xm[m].z; g.w += e[m] * xm[m].w;
                    gq += e[m] * xq[m];
                }
            if (row < dv) {
                float4 r;
                r.x = alpha * s.x + eta * g.x; r.y = alpha * s.y + eta * g.y;
                r.z = alpha * s.z + eta * g.z; r.w = alpha * s.w + eta * g.w;
                *reinterpret_cast<float4 *>(S + (size_t)row * DK + sl * 4) = r;
                if (sl == 0) out[row] = from_f32<T>(alpha * sq + eta * gq);
            }
        }
    }
    // carry: x_prev <- phi(k_t); the window drops its oldest sample and
    // appends the current one (x_prev or phi(k_t), v_t)
    const float inv = knorm > 0.f ? rsqrtf(knorm) : 0.f;
    if (xp)
        for (int i = threadIdx.x; i < DK; i += blockDim.x) xp[i] = kn[i] * inv;
    if (w > 1) {
        for (int i = threadIdx.x; i < (w - 1) * (DK + dv); i += blockDim.x) {
            const int m = i / (DK + dv), c = i % (DK + dv);
            win[i] = c < DK ? xw[m + 1][c] : yw[m + 1][c - DK];
        }
    }
}

// Window-1 variants (Falcon-1/2/1A/2A), the decode hot path.  A row of S is
// held by LPR = min(8, DK/4) lanes, lane l owning float4 slots l, l+LPR, ...
// (every load instruction reads LPR*16 contiguous bytes of a row), so a row's
// dot products need only log2(LPR) shuffle steps; 1/(eps+n), beta and the
// shared sample are staged once per block, never per row.  A block serves
// HPB (n,h) pairs so that the whole grid is resident at once (one wave).
// (n,h) pairs and warps per block of decode1_kernel: at d = 128 one pair per
// block of four warps (eight blocks per SM, so the blocks spread evenly over
// the SMs), below two pairs per block of eight warps (four per SM); either
// way the grid of the decode shapes is resident at once
__host__ __device__ constexpr int decode1_hpb(int dk) { return dk >= 128 ? 1 : 2; }
__host__ __device__ constexpr int decode1_warps(int dk) { return dk >= 128 ? 4 : 8; }

template <typename T, int DK>
__global__ void __launch_bounds__(32 * decode1_warps(DK), DK >= 128 ? 8 : 4) decode1_kernel(DecodeParams p) {
    constexpr int HPB = decode1_hpb(DK);
    constexpr int LPR = DK >= 32 ? 8 : DK / 4;
    constexpr int NV4 = DK / (4 * LPR);  // float4 per lane per row
    constexpr int RPW = 32 / LPR;        // rows per warp per pass
    constexpr int NW = decode1_warps(DK);
    __shared__ __align__(16) float xs[HPB][DK];
    __shared__ __align__(16) float qs[HPB][DK];
    __shared__ float ks[HPB][DK];
    __shared__ float ys[HPB][128];
    __shared__ float bs[HPB][128];
    __shared__ float red[HPB][3][NW];
    __shared__ float hsc[HPB][5];  // inv_den, xq, lambda, |k|^2, 1/|k| (same-step pair)

    const VariantInfo vi = variant_info(p.variant, 1);
    const int nh_total = p.N * p.H, dv = p.dv;
    const int nh0 = blockIdx.x * HPB;
    const int nheads = min(HPB, nh_total - nh0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // below d = 128 the first row of the state is requested before anything
    // else (the staging below then runs under its latency; at d = 128 the
    // row's 16 registers would spill across the staging)
    const int sl = lane % LPR, rsub = warp * RPW + lane / LPR;
    const int total = nheads * dv, stride = NW * RPW;
    float4 cur[NV4], nxt[NV4];
    auto load_row = [&](int r, float4(&dst)[NV4]) {
        if (r < total) {
            const int hh = r / dv, row = r - hh * dv;
            const float4 *Srow = reinterpret_cast<const float4 *>(p.state + ((size_t)(nh0 + hh) * dv + row) * DK);
            // read once per step: evict-first (the row is written back below)
#pragma unroll
            for (int i = 0; i < NV4; ++i) dst[i] = __ldcs(Srow + sl + LPR * i);
        }
    };
    if constexpr (NV4 <= 2) load_row(rsub, cur);

    // stage each pair's sample x = x_prev (prefix pair) or k, normalised
    // below (same-step pair), q, k, v and beta
    const bool same = p.pairing != 0;
    for (int hh = 0; hh < nheads; ++hh) {
        const int nh = nh0 + hh;
        const T *q = static_cast<const T *>(p.q) + (size_t)nh * DK;
        const T *k = static_cast<const T *>(p.k) + (size_t)nh * DK;
        const T *v = static_cast<const T *>(p.v) + (size_t)nh * dv;
        const T *beta = static_cast<const T *>(p.beta) + (size_t)nh * (vi.per_channel ? dv : 1);
        const float *xp = same ? nullptr : p.x_prev + (size_t)nh * DK;
        float px = 0.f, pq = 0.f, pk = 0.f;
        for (int i = threadIdx.x; i < DK; i += blockDim.x) {
            const float qv = to_f32(q[i]), kv = to_f32(k[i]), xv = same ? kv : xp[i];
            xs[hh][i] = xv;
            qs[hh][i] = qv;
            ks[hh][i] = kv;
            px += xv * xv;
            pq += xv * qv;
            pk += kv * kv;
        }
        for (int i = threadIdx.x; i < dv; i += blockDim.x) {
            ys[hh][i] = to_f32(v[i]);
            bs[hh][i] = to_f32(beta[vi.per_channel ? i : 0]);
        }
        px = group_sum<32>(px);
        pq = group_sum<32>(pq);
        pk = group_sum<32>(pk);
        if (lane == 0) { red[hh][0][warp] = px; red[hh][1][warp] = pq; red[hh][2][warp] = pk; }
    }
    __syncthreads();
    if (threadIdx.x < nheads) {
        const int hh = threadIdx.x;
        float n = 0.f, xq = 0.f, knorm = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) { n += red[hh][0][w]; xq += red[hh][1][w]; knorm += red[hh][2][w]; }
        if (same) {  // x = k / |k|: its energy and its product with q
            const float inv = knorm > 0.f ? rsqrtf(knorm) : 0.f;
            n *= inv * inv;
            xq *= inv;
            hsc[hh][4] = inv;
        }
        hsc[hh][0] = n > 0.f ? 1.f / (p.eps + n) : 0.f;  // eta = beta * inv_den
        hsc[hh][1] = xq;
        hsc[hh][2] = p.lambda[(nh0 + hh) % p.H];
        hsc[hh][3] = knorm;
    }
    __syncthreads();
    if (same) {
        for (int hh = 0; hh < nheads; ++hh)
            for (int i = threadIdx.x; i < DK; i += blockDim.x) xs[hh][i] *= hsc[hh][4];
        __syncthreads();
    }

    // the next row's state is loaded before this row is reduced, so two rows'
    // loads are in flight per lane (the step waits on HBM, not on issue)
    if constexpr (NV4 > 2) load_row(rsub, cur);
    for (int r = rsub; r < total; r += stride) {
        load_row(r + stride, nxt);
        const int hh = r / dv, row = r - hh * dv;  // uniform across a row's lanes
        float4 xr[NV4], qr[NV4];
        float4 *Srow = reinterpret_cast<float4 *>(p.state + ((size_t)(nh0 + hh) * dv + row) * DK);
#pragma unroll
        for (int i = 0; i < NV4; ++i) {
            xr[i] = *reinterpret_cast<const float4 *>(&xs[hh][4 * (sl + LPR * i)]);
            qr[i] = *reinterpret_cast<const float4 *>(&qs[hh][4 * (sl + LPR * i)]);
        }
        float sq = 0.f, sx = 0.f;
#pragma unroll
        for (int i = 0; i < NV4; ++i) {
            sq += cur[i].x * qr[i].x + cur[i].y * qr[i].y + cur[i].z * qr[i].z + cur[i].w * qr[i].w;
            sx += cur[i].x * xr[i].x + cur[i].y * xr[i].y + cur[i].z * xr[i].z + cur[i].w * xr[i].w;
        }
        sq = group_sum<LPR>(sq);
        if (vi.regression) sx = group_sum<LPR>(sx);
        const float eta = bs[hh][row] * hsc[hh][0];
        const float alpha = fmaxf(1.f - eta * hsc[hh][2], kAlphaFloor);
        const float e = vi.regression ? ys[hh][row] - sx : ys[hh][row];
        const float ge = eta * e;
#pragma unroll
        for (int i = 0; i < NV4; ++i) {
            float4 o;
            o.x = alpha * cur[i].x + ge * xr[i].x;
            o.y = alpha * cur[i].y + ge * xr[i].y;
            o.z = alpha * cur[i].z + ge * xr[i].z;
            o.w = alpha * cur[i].w + ge * xr[i].w;
            __stcs(Srow + sl + LPR * i, o);  // (streaming: not read again this step)
        }
        if (sl == 0)
            static_cast<T *>(p.out)[(size_t)(nh0 + hh) * dv + row] = from_f32<T>(alpha * sq + ge * hsc[hh][1]);
#pragma unroll
        for (int i = 0; i < NV4; ++i) cur[i] = nxt[i];
    }
    // carry: x_prev <- phi(k_t) (the same-step pair may leave it out)
    for (int hh = 0; hh < nheads && p.x_prev; ++hh) {
        const float kn = hsc[hh][3];
        const float kinv = kn > 0.f ? rsqrtf(kn) : 0.f;
        float *xp = p.x_prev + (size_t)(nh0 + hh) * DK;
        for (int i = threadIdx.x; i < DK; i += blockDim.x) xp[i] = ks[hh][i] * kinv;
    }
}

// Window-1 decode at d = 64 with the state streamed through shared memory:
// one block of four warps per (n,h) pair.  Thread 0 bulk-copies the pair's
// state (16 KB) in four stages of 16 rows, all issued before the block stages
// its token vectors; the lanes read their row from shared memory and store
// the new row straight to HBM.  At d = 64 a pair's rows are few, so
// decode1_kernel's two rows in flight per lane left the step latency-bound
// (15.9 us against 14.3 us here on N = 64, H = 16).  At d = 128 this layout
// measured no faster than decode1_kernel (31.9 against 31.2 us: there the
// step is bound by the HBM read/write mix, not by loads in flight), so d = 128
// keeps decode1_kernel.  The row arithmetic is decode1_kernel's.  Every wait
// is bounded; a give-up leaves the pair's outputs incomplete and is counted.
__device__ unsigned int g_decode_wait_timeouts;

template <typename T, int DK>
__global__ void __launch_bounds__(128, 8) decode1r_kernel(DecodeParams p) {
    constexpr int LPR = 8, NV4 = DK / (4 * LPR), RPW = 32 / LPR, NW = 4;
    constexpr int RPS = NW * RPW;  // rows per stage: 16
    constexpr int NST = 4;  // with d_v <= 64 rows, a pair's whole state
    __shared__ __align__(128) float ring[NST][RPS * DK];
    __shared__ __align__(8) uint64_t bars[NST];
    __shared__ __align__(16) float xs[DK];
    __shared__ __align__(16) float qs[DK];
    __shared__ float ks[DK];
    __shared__ float ys[128];
    __shared__ float bs[128];
    __shared__ float red[3][NW];
    __shared__ float hsc[5];  // inv_den, xq, lambda, |k|^2, 1/|k| (same-step pair)

    const VariantInfo vi = variant_info(p.variant, 1);
    const int nh = blockIdx.x, dv = p.dv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nstage = (dv + RPS - 1) / RPS;
    float *S = p.state + (size_t)nh * dv * DK;
    int issued = 0;  // stages issued (thread 0)
    auto issue = [&](int st) {
        const int rows = min(RPS, dv - st * RPS);
        const uint32_t bytes = (uint32_t)(rows * DK * 4);
        uint64_t *b = &bars[st % NST];
        tc::mbar_arrive_expect_tx(b, bytes);
        tc::bulk_load(tc::smem_u32(ring[st % NST]), S + (size_t)st * RPS * DK, bytes, b);
        ++issued;
    };
    if (tid == 0) {
        for (int i = 0; i < NST; ++i) tc::mbar_init(&bars[i], 1);
        tc::fence_mbar_init();
        for (int st = 0; st < min(NST, nstage); ++st) issue(st);
    }

    // stage the sample x = x_prev (prefix pair) or k, normalised below
    // (same-step pair), q, k, v and beta
    const bool same = p.pairing != 0;
    const T *q = static_cast<const T *>(p.q) + (size_t)nh * DK;
    const T *k = static_cast<const T *>(p.k) + (size_t)nh * DK;
    const T *v = static_cast<const T *>(p.v) + (size_t)nh * dv;
    const T *beta = static_cast<const T *>(p.beta) + (size_t)nh * (vi.per_channel ? dv : 1);
    {
        const float *xp = same ? nullptr : p.x_prev + (size_t)nh * DK;
        float px = 0.f, pq = 0.f, pk = 0.f;
        for (int i = tid; i < DK; i += blockDim.x) {
            const float qv = to_f32(q[i]), kv = to_f32(k[i]), xv = same ? kv : xp[i];
            xs[i] = xv;
            qs[i] = qv;
            ks[i] = kv;
            px += xv * xv;
            pq += xv * qv;
            pk += kv * kv;
        }
        for (int i = tid; i < dv; i += blockDim.x) {
            ys[i] = to_f32(v[i]);
            bs[i] = to_f32(beta[vi.per_channel ? i : 0]);
        }
        px = group_sum<32>(px);
        pq = group_sum<32>(pq);
        pk = group_sum<32>(pk);
        if (lane == 0) { red[0][warp] = px; red[1][warp] = pq; red[2][warp] = pk; }
    }
    __syncthreads();
    if (tid == 0) {
        float n = 0.f, xq = 0.f, knorm = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) { n += red[0][w]; xq += red[1][w]; knorm += red[2][w]; }
        if (same) {  // x = k / |k|: its energy and its product with q
            const float inv = knorm > 0.f ? rsqrtf(knorm) : 0.f;
            n *= inv * inv;
            xq *= inv;
            hsc[4] = inv;
        }
        hsc[0] = n > 0.f ? 1.f / (p.eps + n) : 0.f;  // eta = beta * inv_den
        hsc[1] = xq;
        hsc[2] = p.lambda[nh % p.H];
        hsc[3] = knorm;
    }
    __syncthreads();
    if (same) {
        for (int i = tid; i < DK; i += blockDim.x) xs[i] *= hsc[4];
        __syncthreads();
    }

    const int sl = lane % LPR, rsub = warp * RPW + lane / LPR;
    float4 xr[NV4], qr[NV4];
#pragma unroll
    for (int i = 0; i < NV4; ++i) {
        xr[i] = *reinterpret_cast<const float4 *>(&xs[4 * (sl + LPR * i)]);
        qr[i] = *reinterpret_cast<const float4 *>(&qs[4 * (sl + LPR * i)]);
    }
    const float inv_den = hsc[0], xq = hsc[1], lam = hsc[2];
    bool ok = true;
    int first_bad = nstage;  // the first stage whose wait gave up
    for (int st = 0; st < nstage; ++st) {
        const int slot = st % NST;
        if (ok) {
            ok = tc::mbar_wait_timeout(&bars[slot], (uint32_t)(st / NST) & 1u, 2000000000ull);
            if (!ok) first_bad = st;
        }
        const int row = st * RPS + rsub;
        if (ok && row < dv) {
            const float4 *src = reinterpret_cast<const float4 *>(&ring[slot][rsub * DK]);
            float4 cur[NV4];
#pragma unroll
            for (int i = 0; i < NV4; ++i) cur[i] = src[sl + LPR * i];
            float sq = 0.f, sx = 0.f;
#pragma unroll
            for (int i = 0; i < NV4; ++i) {
                sq += cur[i].x * qr[i].x + cur[i].y * qr[i].y + cur[i].z * qr[i].z + cur[i].w * qr[i].w;
                sx += cur[i].x * xr[i].x + cur[i].y * xr[i].y + cur[i].z * xr[i].z + cur[i].w * xr[i].w;
            }
            sq = group_sum<LPR>(sq);
            if (vi.regression) sx = group_sum<LPR>(sx);
            const float eta = bs[row] * inv_den;
            const float alpha = fmaxf(1.f - eta * lam, kAlphaFloor);
            const float y = ys[row];
            const float ge = eta * (vi.regression ? y - sx : y);
            float4 *dst = reinterpret_cast<float4 *>(S + (size_t)row * DK);
#pragma unroll
            for (int i = 0; i < NV4; ++i) {
                float4 o;
                o.x = alpha * cur[i].x + ge * xr[i].x;
                o.y = alpha * cur[i].y + ge * xr[i].y;
                o.z = alpha * cur[i].z + ge * xr[i].z;
                o.w = alpha * cur[i].w + ge * xr[i].w;
                dst[sl + LPR * i] = o;
            }
            if (sl == 0) static_cast<T *>(p.out)[(size_t)nh * dv + row] = from_f32<T>(alpha * sq + ge * xq);
        }
        // every thread has read the stage: it may be written again
        tc::fence_proxy_async();
        __syncthreads();
        if (tid == 0 && ok && st + NST < nstage) issue(st + NST);
    }
    // carry: x_prev <- phi(k_t) (the same-step pair may leave it out)
    if (p.x_prev) {
        const float kn = hsc[3];
        const float kinv = kn > 0.f ? rsqrtf(kn) : 0.f;
        for (int i = tid; i < DK; i += blockDim.x) p.x_prev[(size_t)nh * DK + i] = ks[i] * kinv;
    }
    if (tid == 0 && !ok) {
        atomicAdd(&g_decode_wait_timeouts, 1u);
        // copies still in flight (from the stage that gave up on) must land
        // before the block leaves
        for (int st = first_bad; st < issued; ++st)
            (void)tc::mbar_wait_timeout(&bars[st % NST], (uint32_t)(st / NST) & 1u, 2000000000ull);
    }
}

// Window variants (Falcon-3/3A, W = 2..8 samples per update), laid out as
// decode1_kernel: LPR lanes per row of S, HPB (n,h) pairs per block so the
// whole grid is resident at once, and the first rows of the state requested
// before the block stages its window.  Per row: W + 1 dot products (S_j.x_m,
// S_j.q) reduced together, e_m = y_m - S_j.x_m (inner product: y_m), and
// S_j <- alpha S_j + eta sum_m e_m x_m^T, o_j = alpha S_j.q + eta sum_m e_m (x_m.q).
// At d = 128 one pair per block of four warps, seven blocks per SM (so the
// blocks spread evenly and 32 warps per SM keep rows in flight); below, four
// pairs per block of eight warps, two blocks per SM.
__host__ __device__ constexpr int decodew_hpb(int dk) { return dk >= 128 ? 1 : 4; }
__host__ __device__ constexpr int decodew_warps(int dk) { return dk >= 128 ? 4 : 8; }

template <typename T, int DK, int W>
__global__ void __launch_bounds__(32 * decodew_warps(DK), DK >= 128 ? 7 : 2) decodew_kernel(DecodeParams p) {
    constexpr int HPB = decodew_hpb(DK);
    constexpr int LPR = DK >= 32 ? 8 : DK / 4;
    constexpr int NV4 = DK / (4 * LPR);  // float4 per lane per row
    constexpr int RPW = 32 / LPR;        // rows per warp per pass
    constexpr int NW = decodew_warps(DK);
    __shared__ __align__(16) float xs[HPB][W][DK];  // samples, oldest first; slot W-1 the current one
    __shared__ __align__(16) float qs[HPB][DK];
    __shared__ float ks[HPB][DK];
    __shared__ float ys[HPB][W][128];
    __shared__ float red[HPB][W + 1][2];  // per sample |x_m|^2 and x_m.q; then |k|^2
    __shared__ float hsc[HPB][W + 3];     // eta, alpha, 1/|k|, x_m.q for m < W

    const bool reg = variant_info(p.variant, W).regression;
    const int nh_total = p.N * p.H, dv = p.dv;
    const int nh0 = blockIdx.x * HPB;
    const int nheads = min(HPB, nh_total - nh0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool same = p.pairing != 0;  // same-step pair: the current sample is (phi(k_t), v_t)

    const int sl = lane % LPR, rsub = warp * RPW + lane / LPR;
    const int total = nheads * dv, stride = NW * RPW;
    float4 cur[NV4], nxt[NV4];
    auto load_row = [&](int r, float4(&dst)[NV4]) {
        if (r < total) {
            const int hh = r / dv, row = r - hh * dv;
            const float4 *Srow = reinterpret_cast<const float4 *>(p.state + ((size_t)(nh0 + hh) * dv + row) * DK);
#pragma unroll
            for (int i = 0; i < NV4; ++i) dst[i] = __ldcs(Srow + sl + LPR * i);  // read once: evict first
        }
    };
    load_row(rsub, cur);
    load_row(rsub + stride, nxt);

    // stage the window (oldest first), the current sample (x_prev, or k to be
    // normalised under the same-step pair), q and k
    for (int hh = 0; hh < nheads; ++hh) {
        const int nh = nh0 + hh;
        const T *q = static_cast<const T *>(p.q) + (size_t)nh * DK;
        const T *k = static_cast<const T *>(p.k) + (size_t)nh * DK;
        const T *v = static_cast<const T *>(p.v) + (size_t)nh * dv;
        const float *xp = p.x_prev ? p.x_prev + (size_t)nh * DK : nullptr;
        const float *win = p.win + (size_t)nh * (W - 1) * (DK + dv);
        for (int i = threadIdx.x; i < DK; i += blockDim.x) {
            const float kv = to_f32(k[i]);
            qs[hh][i] = to_f32(q[i]);
            ks[hh][i] = kv;
            xs[hh][W - 1][i] = same ? kv : xp[i];
        }
        for (int i = threadIdx.x; i < dv; i += blockDim.x) ys[hh][W - 1][i] = to_f32(v[i]);
        for (int i = threadIdx.x; i < (W - 1) * (DK + dv); i += blockDim.x) {
            const int m = i / (DK + dv), c = i % (DK + dv);
            const float val = win[i];
            if (c < DK) xs[hh][m][c] = val; else ys[hh][m][c - DK] = val;
        }
    }
    __syncthreads();
    // one warp per (pair, sample): |x_m|^2 and x_m.q; job m = W: |k|^2
    for (int job = warp; job < nheads * (W + 1); job += NW) {
        const int hh = job / (W + 1), m = job % (W + 1);
        const float *x = m < W ? xs[hh][m] : ks[hh];
        float a = 0.f, b = 0.f;
        for (int c = lane; c < DK; c += 32) {
            a += x[c] * x[c];
            b += x[c] * qs[hh][c];
        }
        a = group_sum<32>(a);
        b = group_sum<32>(b);
        if (lane == 0) { red[hh][m][0] = a; red[hh][m][1] = b; }
    }
    __syncthreads();
    if (threadIdx.x < nheads) {
        const int hh = threadIdx.x;
        const float knorm = red[hh][W][0];
        const float kinv = knorm > 0.f ? rsqrtf(knorm) : 0.f;
        float n = 0.f;
#pragma unroll
        for (int m = 0; m < W; ++m) {
            float e2 = red[hh][m][0], xq = red[hh][m][1];
            if (same && m == W - 1) {  // x = k / |k|
                e2 *= kinv * kinv;
                xq *= kinv;
            }
            n += e2;
            hsc[hh][3 + m] = xq;
        }
        const float lam = p.lambda[(nh0 + hh) % p.H];
        float eta, alpha;
        step_and_decay(to_f32(static_cast<const T *>(p.beta)[nh0 + hh]), n, p.eps, lam, eta, alpha);
        hsc[hh][0] = eta;
        hsc[hh][1] = alpha;
        hsc[hh][2] = kinv;
    }
    __syncthreads();
    if (same) {
        for (int hh = 0; hh < nheads; ++hh)
            for (int i = threadIdx.x; i < DK; i += blockDim.x) xs[hh][W - 1][i] *= hsc[hh][2];
        __syncthreads();
    }

    for (int r = rsub; r < total; r += stride) {
        const int hh = r / dv, row = r - hh * dv;  // uniform across a row's lanes
        float4 *Srow = reinterpret_cast<float4 *>(p.state + ((size_t)(nh0 + hh) * dv + row) * DK);
        float sq = 0.f, sx[W];
#pragma unroll
        for (int m = 0; m < W; ++m) sx[m] = 0.f;
#pragma unroll
        for (int i = 0; i < NV4; ++i) {
            const float4 q4 = *reinterpret_cast<const float4 *>(&qs[hh][4 * (sl + LPR * i)]);
            sq += cur[i].x * q4.x + cur[i].y * q4.y + cur[i].z * q4.z + cur[i].w * q4.w;
            if (reg) {
#pragma unroll
                for (int m = 0; m < W; ++m) {
                    const float4 x4 = *reinterpret_cast<const float4 *>(&xs[hh][m][4 * (sl + LPR * i)]);
                    sx[m] += cur[i].x * x4.x + cur[i].y * x4.y + cur[i].z * x4.z + cur[i].w * x4.w;
                }
            }
        }
        sq = group_sum<LPR>(sq);
        const float eta = hsc[hh][0], alpha = hsc[hh][1];
        float ge[W], gq = 0.f;
#pragma unroll
        for (int m = 0; m < W; ++m) {
            const float e = reg ? ys[hh][m][row] - group_sum<LPR>(sx[m]) : ys[hh][m][row];
            ge[m] = eta * e;
            gq += ge[m] * hsc[hh][3 + m];
        }
#pragma unroll
        for (int i = 0; i < NV4; ++i) {
            float4 o;
            o.x = alpha * cur[i].x; o.y = alpha * cur[i].y; o.z = alpha * cur[i].z; o.w = alpha * cur[i].w;
#pragma unroll
            for (int m = 0; m < W; ++m) {
                const float4 x4 = *reinterpret_cast<const float4 *>(&xs[hh][m][4 * (sl + LPR * i)]);
                o.x += ge[m] * x4.x; o.y += ge[m] * x4.y; o.z += ge[m] * x4.z; o.w += ge[m] * x4.w;
            }
            __stcs(Srow + sl + LPR * i, o);  // streaming store
        }
        if (sl == 0) static_cast<T *>(p.out)[(size_t)(nh0 + hh) * dv + row] = from_f32<T>(alpha * sq + gq);
#pragma unroll
        for (int i = 0; i < NV4; ++i) cur[i] = nxt[i];
        load_row(r + 2 * stride, nxt);
    }
    // carry: x_prev <- phi(k_t); the window drops its oldest sample and
    // appends the current one
    for (int hh = 0; hh < nheads; ++hh) {
        const int nh = nh0 + hh;
        if (p.x_prev)
            for (int i = threadIdx.x; i < DK; i += blockDim.x) p.x_prev[(size_t)nh * DK + i] = ks[hh][i] * hsc[hh][2];
        float *win = p.win + (size_t)nh * (W - 1) * (DK + dv);
        for (int i = threadIdx.x; i < (W - 1) * (DK + dv); i += blockDim.x) {
            const int m = i / (DK + dv), c = i % (DK + dv);
            win[i] = c < DK ? xs[hh][m + 1][c] : ys[hh][m + 1][c - DK];
        }
    }
}

template <typename T, int DK>
__global__ void __launch_bounds__(128) carry_kernel(CarryParams p) {
    const VariantInfo vi = variant_info(p.variant, p.window);
    const int w = vi.window;
    const int bh = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T *k = static_cast<const T *>(p.k) + (size_t)bh * p.L * DK;
    const T *v = static_cast<const T *>(p.v) + (size_t)bh * p.L * p.dv;
    // job 0: x_prev = phi(k_L); jobs 1..w-1: window slots m = job-1, the
    // samples i = L-w+1+m (0-based) whose key is k_{i-1} (prefix pair) or k_i
    // (same-step pair)
    for (int job = warp; job < w; job += 4) {
        if (job == 0 && !p.x_prev) continue;
        const int m = job - 1;
        const int i = job == 0 ? p.L : p.L - (w - 1) + m;
        float *xdst = job == 0 ? p.x_prev + (size_t)bh * DK : p.win + ((size_t)bh * (w - 1) + m) * (DK + p.dv);
        const int ki = (job > 0 && p.pairing != 0) ? i : i - 1;
        float ss = 0.f;
        for (int c = lane; c < DK; c += 32) {
            const float x = (ki >= 0 && i >= 0) ? to_f32(k[(size_t)ki * DK + c]) : 0.f;
            ss += x * x;
        }
        ss = group_sum<32>(ss);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
        for (int c = lane; c < DK; c += 32)
            xdst[c] = (ki >= 0 && i >= 0) ? to_f32(k[(size_t)ki * DK + c]) * inv : 0.f;
        if (job > 0)
            for (int c = lane; c < p.dv; c += 32)
                xdst[DK + c] = i >= 0 ? to_f32(v[(size_t)i * p.dv + c]) : 0.f;
    }
}

template <typename T, int DK, int W>
static void launch_decodew(const DecodeParams &p, cudaStream_t s) {
    constexpr int hpb = decodew_hpb(DK);
    decodew_kernel<T, DK, W><<<(p.N * p.H + hpb - 1) / hpb, 32 * decodew_warps(DK), 0, s>>>(p);
}

template <typename T, int DK>
static void launch_decode_dk(const DecodeParams &p, cudaStream_t s) {
    switch (variant_info(p.variant, p.window).window) {
        case 1: {
            if constexpr (DK == 64) {
                // bulk copies need a 16-byte aligned state; more than 64 value
                // rows would need more stages than the ring holds
                if ((reinterpret_cast<uintptr_t>(p.state) & 15u) == 0 && p.dv <= 64) {
                    decode1r_kernel<T, DK><<<p.N * p.H, 128, 0, s>>>(p);
                    return;
                }
            }
            constexpr int hpb = decode1_hpb(DK);
            decode1_kernel<T, DK><<<(p.N * p.H + hpb - 1) / hpb, 32 * decode1_warps(DK), 0, s>>>(p);
            return;
        }
        case 2: launch_decodew<T, DK, 2>(p, s); return;
        case 3: launch_decodew<T, DK, 3>(p, s); return;
        case 4: launch_decodew<T, DK, 4>(p, s); return;
        default: decode_kernel<T, DK><<<p.N * p.H, 256, 0, s>>>(p); return;  // windows 5-8
    }
}

template <typename T>
int launch_decode(const DecodeParams &p, cudaStream_t s) {
    switch (p.dk) {
        case 16: launch_decode_dk<T, 16>(p, s); return 0;
        case 32: launch_decode_dk<T, 32>(p, s); return 0;
        case 64: launch_decode_dk<T, 64>(p, s); return 0;
        case 128: launch_decode_dk<T, 128>(p, s); return 0;
    }
    return -3;
}

template <typename T>
int launch_carry(const CarryParams &p, cudaStream_t s) {
    switch (p.dk) {
        case 16: carry_kernel<T, 16><<<p.B * p.H, 128, 0, s>>>(p); return 0;
        case 32: carry_kernel<T, 32><<<p.B * p.H, 128, 0, s>>>(p); return 0;
        case 64: carry_kernel<T, 64><<<p.B * p.H, 128, 0, s>>>(p); return 0;
        case 128: carry_kernel<T, 128><<<p.B * p.H, 128, 0, s>>>(p); return 0;
    }
    return -3;
}

unsigned int decode_wait_timeouts() {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_decode_wait_timeouts, sizeof(v));
    return v;
}

template int launch_decode<float>(const DecodeParams &, cudaStream_t);
template int launch_decode<__nv_bfloat16>(const DecodeParams &, cudaStream_t);
template int launch_carry<float>(const CarryParams &, cudaStream_t);
template int launch_carry<__nv_bfloat16>(const CarryParams &, cudaStream_t);

}  // namespace falcon
