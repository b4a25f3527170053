// warp_tf32.cuh -- 64 x 64 fp32 shared-memory tile products on the TF32 warp
// MMAs (mma.sync m16n8k8, fp32 accumulation) for blocks of 8 or 16 warps: the
// operand and accumulator conventions of the chunk-backward and the
// masked-parallel kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tc_sm100.cuh"

namespace falcon {
namespace wt {

// an fp32 value as a TF32 operand: the tensor core reads its top 19 bits
__device__ __forceinline__ uint32_t tf(float x) { return __float_as_uint(x); }

// The m16n8k8 TF32 slots of one 8-wide slice of k are filled in the order
// slot t <- k0 + 2t, slot t + 4 <- k0 + 2t + 1 (lane quad t = 0..3), for A
// and B alike: the slice's sum is unchanged, and a row-major operand gives
// both of a lane's values in one 8-byte load.
//
// C += op(A) op(B) over kb <= k < ke (multiples of 8) for this warp's 16 x 8NT
// block (rows 16 (w & 3), columns 8NT (w >> 2)) of a 64 x 64 result: NT = 4
// for a block of eight warps, 2 for sixteen.  Tiles of row stride LD (even).
// op(A)(r, k) = TA ? A[k][r] : A[r][k], times sk[k] when SK;
// op(B)(k, n) = TB ? B[n][k] : B[k][n].
template <int LD, bool TA, bool TB, bool SK = false, int NT = 4>
__device__ __forceinline__ void mma64(const float *A, const float *B, float (&acc)[NT][4], int kb, int ke,
                                      const float *sk = nullptr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
    const int rb = (warp & 3) * 16, cb = (warp >> 2) * 8 * NT;
#pragma unroll 2
    for (int k0 = kb; k0 < ke; k0 += 8) {
        const int ka = k0 + 2 * t;
        float a0, a1, a2, a3;  // (r, ka), (r + 8, ka), (r, ka + 1), (r + 8, ka + 1), r = rb + g
        if (TA) {
            a0 = A[ka * LD + rb + g];
            a1 = A[ka * LD + rb + g + 8];
            a2 = A[(ka + 1) * LD + rb + g];
            a3 = A[(ka + 1) * LD + rb + g + 8];
        } else {
            const float2 u0 = *reinterpret_cast<const float2 *>(A + (rb + g) * LD + ka);
            const float2 u1 = *reinterpret_cast<const float2 *>(A + (rb + g + 8) * LD + ka);
            a0 = u0.x; a2 = u0.y; a1 = u1.x; a3 = u1.y;
        }
        if (SK) {
            const float2 s = *reinterpret_cast<const float2 *>(sk + ka);
            a0 *= s.x; a1 *= s.x; a2 *= s.y; a3 *= s.y;
        }
        const uint32_t a[4] = {tf(a0), tf(a1), tf(a2), tf(a3)};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = cb + nt * 8 + g;
            uint32_t b[2];
            if (TB) {
                const float2 v = *reinterpret_cast<const float2 *>(B + n * LD + ka);
                b[0] = tf(v.x);
                b[1] = tf(v.y);
            } else {
                b[0] = tf(B[ka * LD + n]);
                b[1] = tf(B[(ka + 1) * LD + n]);
            }
            tc::mma_tf32(acc[nt], a, b);
        }
    }
}

template <int NT>
__device__ __forceinline__ void zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
}

// f(row, col, value&) over this warp's accumulator elements
template <int NT, typename Fn>
__device__ __forceinline__ void each(float (&acc)[NT][4], Fn f) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
    const int rb = (warp & 3) * 16, cb = (warp >> 2) * 8 * NT;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) f(rb + g + (e >> 1) * 8, cb + nt * 8 + 2 * t + (e & 1), acc[nt][e]);
}

// eight bf16 (one 16-byte piece) to eight fp32 in shared memory (16-byte aligned)
__device__ __forceinline__ void st8(float *dst, const uint4 &w) {
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
    float4 lo, hi;
    lo.x = __uint_as_float(x[0] << 16); lo.y = __uint_as_float(x[0] & 0xffff0000u);
    lo.z = __uint_as_float(x[1] << 16); lo.w = __uint_as_float(x[1] & 0xffff0000u);
    hi.x = __uint_as_float(x[2] << 16); hi.y = __uint_as_float(x[2] & 0xffff0000u);
    hi.z = __uint_as_float(x[3] << 16); hi.w = __uint_as_float(x[3] & 0xffff0000u);
    reinterpret_cast<float4 *>(dst)[0] = lo;
    reinterpret_cast<float4 *>(dst)[1] = hi;
}

__device__ __forceinline__ uint4 ld16(const void *p) { return *reinterpret_cast<const uint4 *>(p); }

}  // namespace wt
}  // namespace falcon
