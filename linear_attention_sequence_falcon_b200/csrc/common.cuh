// common.cuh -- device helpers shared by the Falcon kernels (sm_100a).
//
// Method: Falcon normalised first-order fast-weight updates, from the pages
// "Fast Weight Attention：用于持续学习的快速权重注意力" (核心方法 1-4),
// "Fast Weight Attention for Continual Learning" (方法) and
// "借鉴40年前的设想！字节Seed提出快速权重注意力推进大模型持续学习" (02).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace falcon {

// Positive-decay floor: alpha = max(1 - eta*lambda, 2^-20).
constexpr float kAlphaFloor = 9.5367431640625e-07f;
constexpr int kMaxWindow = 8;

enum Variant { F1 = 0, F2 = 1, F3 = 2, F1A = 3, F2A = 4, F3A = 5 };

struct VariantInfo {
    bool regression;   // squared-error objective (erase step) vs inner product
    bool per_channel;  // one step per value channel (Falcon-2/2A)
    int window;        // samples per update (Falcon-3/3A: B_w, else 1)
};

__host__ __device__ inline VariantInfo variant_info(int v, int window) {
    VariantInfo vi;
    vi.regression = (v == F1 || v == F2 || v == F3);
    vi.per_channel = (v == F2 || v == F2A);
    vi.window = (v == F3 || v == F3A) ? window : 1;
    return vi;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// NLMS step and positive decay for one sample with energy n (reading: an
// empty sample, n == 0, takes no step and no decay).
__device__ __forceinline__ void step_and_decay(float beta, float n, float eps, float lambda,
                                               float &eta, float &alpha) {
    eta = n > 0.f ? beta / (eps + n) : 0.f;
    alpha = fmaxf(1.f - eta * lambda, kAlphaFloor);
}

template <int W>
__device__ __forceinline__ float group_sum(float x) {
    // xor-reduction inside aligned groups of W lanes
#pragma unroll
    for (int o = W / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace falcon
