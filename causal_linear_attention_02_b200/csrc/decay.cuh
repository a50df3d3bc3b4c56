// Per-head decay on the state, and the elementwise feature map.
//
// Decay (not on the pages: the Lightning Attention-2 form of the same method,
// taken in its plainest reading; a rate of 1 is the method without decay):
//   S_t = lambda_h S_{t-1} + k_t^T v_t,   S_{start-1} = S0,   o_t = q_t S_t,
// so that for a block of n tokens starting at b0, with KV the state just before
// b0 and r = t - b0:
//   O_t  = sum_{u = b0..t} lambda^(t-u) (q_t . k_u) v_u  +  lambda^(r+1) q_t KV,
//   KV' = lambda^n KV + sum_u lambda^(b0+n-1-u) k_u^T v_u.
// Rates are fp32 [H] in device memory. A rate outside [0, 1] (or NaN) records
// LA_ERR_BAD_DECAY: decay_check_kernel empties a prefill call's work list, and
// each kernel also skips a head whose rate it finds bad.
//
// Feature map (page "MiniMax-M2.5语言模型：Linear Attention架构解析与实践",
// section "2.2 Linear Attention的数学原理", alpha = 0.3 there):
//   phi(x) = ELU(x) + alpha x,  ELU(x) = x for x > 0, e^x - 1 otherwise.
#pragma once

#include "common.cuh"

namespace la {

// log2(lambda_h) of one head, after checking the rate (-inf for lambda = 0).
__device__ __forceinline__ bool load_decay(const float* decay, int h, float& log2_lam) {
    const float lam = decay[h];
    if (!(lam >= 0.f && lam <= 1.f)) {
        record_status(LA_ERR_BAD_DECAY);
        return false;
    }
    log2_lam = log2f(lam);
    return true;
}

// lambda^n for an integer n >= 0, from log2(lambda); lambda^0 = 1 also for lambda = 0.
__device__ __forceinline__ float decay_pow(float log2_lam, int n) {
    return n == 0 ? 1.f : exp2f((float)n * log2_lam);
}

// Checks the H rates of a prefill call before its kernels run: a rate outside
// [0, 1] or NaN records LA_ERR_BAD_DECAY and empties the call's work list
// (ctrl->ok = 0, no blocks), so nothing is written. One CTA.
__global__ void __launch_bounds__(256) decay_check_kernel(const float* decay, int H, Control* ctrl) {
    bool bad = false;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        const float x = decay[i];
        bad |= !(x >= 0.f && x <= 1.f);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) {
        record_status(LA_ERR_BAD_DECAY);
        ctrl->ok = 0;
        ctrl->nblocks = 0;
    }
}

__device__ __forceinline__ float phi(float x, float alpha) {
    return (x > 0.f ? x : expm1f(x)) + alpha * x;
}

// y = phi(x) over n elements; 16-byte groups (8 bf16 or 4 fp32) per thread and
// iteration, grid-stride, then the last n mod group elements one by one.
// x and y are 16-byte aligned; y may be x.
template <typename T>
__global__ void __launch_bounds__(256) feature_map_kernel(const T* x, T* y, int64_t n, float alpha) {
    constexpr int G = 16 / sizeof(T);
    const int64_t groups = n / G;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t i = tid; i < groups; i += stride) {
        uint4 w = *reinterpret_cast<const uint4*>(x + i * G);
        if constexpr (sizeof(T) == 4) {
            w.x = __float_as_uint(phi(__uint_as_float(w.x), alpha));
            w.y = __float_as_uint(phi(__uint_as_float(w.y), alpha));
            w.z = __float_as_uint(phi(__uint_as_float(w.z), alpha));
            w.w = __float_as_uint(phi(__uint_as_float(w.w), alpha));
        } else {
            uint32_t* p = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float lo = __uint_as_float(p[j] << 16), hi = __uint_as_float(p[j] & 0xffff0000u);
                p[j] = pack_bf16x2(phi(lo, alpha), phi(hi, alpha));
            }
        }
        *reinterpret_cast<uint4*>(y + i * G) = w;
    }
    for (int64_t i = groups * G + tid; i < n; i += stride) io<T>::st(y + i, phi(io<T>::ld(x + i), alpha));
}

}  // namespace la
