// tc128.cuh -- shared pieces of the d = 128 tensor-core chunk kernels
// (bf16 inputs, d_k = d_v = 128, chunk 64): tile geometry, tcgen05 product
// issue over 128-byte-swizzled K-major tiles, ldmatrix/stmatrix transposes,
// TMA tensor maps of [B*H][L][128] tensors and the sample stage
// x_t = phi(k_{t-1}) with |x_t|^2.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc_sm100.cuh"

namespace falcon {
namespace {

constexpr int CH = 64;    // chunk
constexpr int DD = 128;   // d_k = d_v
constexpr int NTH = 256;
constexpr int ISSUER = 128;
constexpr uint32_t TILE = 8192;                // 64 rows x 128 bytes
constexpr uint32_t SIMG = 4 * TILE;            // bf16 S_c: two K halves of 128 rows x 64
constexpr uint64_t kWaitNs = 2000000000ull;

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

// element (r, c) of a 64-row bf16 tile pair: two 64-column halves, the
// second `hs` bytes after the first
__device__ __forceinline__ uint32_t pair_off(int r, int c, uint32_t hs = TILE) {
    return (uint32_t)(c >> 6) * hs + tc::sw128(r, (c & 63) >> 3) + (uint32_t)(c & 7) * 2;
}

// D (+)= A B^T over K = 64 * nk (4 K=16 slices per 64-column tile), both
// operands K-major 128-byte-swizzled; the k-th K tile of A (B) starts
// a_step (b_step) bytes after the previous one; M = 128.
__device__ __forceinline__ void issue_gemm(uint32_t d_tmem, uint32_t a, uint32_t a_step, uint32_t b,
                                           uint32_t b_step, int nk, int N) {
    const uint32_t idesc = tc::idesc_bf16(128, N, 0, 0);
    for (int kt = 0; kt < nk; ++kt)
        tc::mma_k64(d_tmem, tc::sdesc_sw128(a + kt * a_step, 16, 1024), tc::sdesc_sw128(b + kt * b_step, 16, 1024),
                    idesc, kt > 0);
}

// Transposed copy of four 8x8 blocks of a 64-row bf16 tile (128-byte rows,
// 128-byte swizzle): source row block rb, 16-byte chunks cb0..cb0+3 ->
// destination rows 8*(cb0..cb0+3) (+ dst_row0), chunk rb.  Whole warp.
__device__ __forceinline__ void transpose4(uint32_t src, int rb, int cb0, uint32_t dst, int dst_row0) {
    const int lane = threadIdx.x & 31, m = lane >> 3, i = lane & 7;
    uint32_t r[4];
    tc::ldsm_x4_trans(src + (uint32_t)(rb * 8 + i) * 128u + ((uint32_t)((cb0 + m) ^ i) << 4), r);
    const int drow = dst_row0 + (cb0 + m) * 8 + i;
    tc::stsm_x4(dst + (uint32_t)drow * 128u + ((uint32_t)(rb ^ (drow & 7)) << 4), r);
}

// Transpose a 64 x 128 tile pair (rows s, two 64-column halves) into a
// 128-row K-major tile (rows c, 64 columns s): 32 groups of 4 blocks over
// the block's 8 warps.
__device__ __forceinline__ void transpose_pair(uint32_t src_pair, uint32_t dst128) {
    const int warp = threadIdx.x >> 5;
    for (int g = warp; g < 32; g += NTH / 32) {
        const int half = g >> 4, rb = (g >> 1) & 7, cb0 = (g & 1) * 4;
        transpose4(src_pair + half * TILE, rb, cb0, dst128, half * 64);
    }
}

struct PcMaps {
    CUtensorMap q, k, v, beta;
};

// TMA: a 64-row x 128-column bf16 slab (rows y.., the two halves) into a tile pair
__device__ __forceinline__ void load_pair(uint32_t dst, const CUtensorMap *m, int y, int bh, uint64_t *bar) {
    tc::tma_load_3d(dst, m, 0, y, bh, bar);
    tc::tma_load_3d(dst + TILE, m, 64, y, bh, bar);
}

// samples x_t = phi(k_{t-1}) in place over the raw-key tile pair (four
// threads per row, 32 columns each), |x_t|^2 -> sqn[t].  The first token of
// a continued segment takes the carried phi(k) as given.
__device__ __forceinline__ void samples_pair(uint8_t *sm, uint32_t offx, uint32_t hs, const FwdParams &p, int bh,
                                             bool first_chunk, float *sqn, float *rinv = nullptr) {
    const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
    const bool carried = first_chunk && r == 0 && p.x_prev != nullptr && p.pairing == 0;
    float xr[32];
    float ss = 0.f;
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
        const int c = part * 32 + c8 * 8;
        if (carried) {
#pragma unroll
            for (int e = 0; e < 8; ++e) xr[c8 * 8 + e] = p.x_prev[(size_t)bh * DD + c + e];
        } else {
            unpack8(*reinterpret_cast<const uint4 *>(sm + offx + pair_off(r, c, hs)), &xr[c8 * 8]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += xr[c8 * 8 + e] * xr[c8 * 8 + e];
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const float inv = (carried || p.phi != 0) ? 1.f : (ss > 0.f ? rsqrtf(ss) : 0.f);
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) xr[c8 * 8 + e] *= inv;
        *reinterpret_cast<uint4 *>(sm + offx + pair_off(r, part * 32 + c8 * 8, hs)) = pack8(&xr[c8 * 8]);
    }
    if (part == 0) {
        const float n = ss * inv * inv;
        sqn[r] = n;
        if (rinv) rinv[r] = n > 0.f ? 1.f / (p.eps + n) : 0.f;  // eta_t = beta_t / (eps + |x_t|^2), 0 at x_t = 0
    }
}

// bf16 element (r, c) of a tile pair
__device__ __forceinline__ float pair_get(const uint8_t *sm, uint32_t off, int r, int c) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + off + pair_off(r, c)));
}

}  // namespace

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

// [B*H][L][128] bf16 tensor, boxes of 64 rows x 64 columns (one 128-byte
// swizzled half), zero fill outside.
bool make_map(CUtensorMap *m, const void *base, int BH, int L) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DD, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)DD * 2, (cuuint64_t)L * DD * 2};
    const cuuint32_t box[3] = {64, CH, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

}  // namespace falcon
