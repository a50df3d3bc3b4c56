// Exclusive prefix of per-rank states for sequence parallelism (LASP+).
//
// Each of W ranks holds a contiguous segment of the same sequences. The
// right product only needs, at the start of rank r's segment, the state of
// everything before it, S0 + sum_{r' < r} U_{r'}, where U_{r'} = sum over
// rank r' tokens of k^T v. The ranks therefore exchange their d x d segment
// states with one all-gather and each takes a local prefix sum, in place of a
// serial send/receive chain (page "MiniMax-01 Lightning Attention", section
// "计算优化", item 3; page "首个线性注意力架构的大模型来了…", section "4.2
// 计算优化"). HBM-bound elementwise sum: one 16-byte group per thread and
// iteration, rank order 0, 1, ..., rank-1.
#pragma once

#include "common.cuh"
#include "decay.cuh"

namespace la {

__global__ void __launch_bounds__(256)
state_prefix_kernel(const float4* __restrict__ gathered, int rank, int64_t per_rank4,
                    const float4* init, float4* out) {
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_rank4; i += step) {
        float4 acc = init ? init[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < rank; ++r) {
            const float4 x = __ldcs(gathered + (int64_t)r * per_rank4 + i);
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        out[i] = acc;
    }
}

// With a decay rate per head on the state (decay.cuh), rank r's starting state
// is P_r = lambda_h^(n_{r-1}) P_{r-1} + S_{r-1}, P_0 = S0, where S_{r'} is rank
// r''s segment state (itself decayed to the segment's end) and n_{r'} the
// length of rank r''s segment of the sequence. seg_lens: [world][nseq] int32.
// A bad rate (LA_ERR_BAD_DECAY) or a negative length (LA_ERR_BAD_SEQLENS)
// leaves that state unwritten.
__global__ void __launch_bounds__(256)
state_prefix_decay_kernel(const float4* __restrict__ gathered, const int32_t* __restrict__ seg_lens, int rank,
                          int nseq, int H, int64_t per_state4, int64_t per_rank4, const float* decay,
                          const float4* init, float4* out) {
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_rank4; i += step) {
        const int64_t pair = i / per_state4;              // (sequence, head)
        const int s = (int)(pair / H), h = (int)(pair % H);
        float l2;
        if (!load_decay(decay, h, l2)) continue;
        float4 acc = init ? init[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        bool ok = true;
        for (int r = 0; r < rank; ++r) {
            const int n = seg_lens[(int64_t)r * nseq + s];
            if (n < 0) {
                ok = false;
                break;
            }
            const float w = decay_pow(l2, n);
            const float4 x = __ldcs(gathered + (int64_t)r * per_rank4 + i);
            acc.x = fmaf(w, acc.x, x.x);
            acc.y = fmaf(w, acc.y, x.y);
            acc.z = fmaf(w, acc.z, x.z);
            acc.w = fmaf(w, acc.w, x.w);
        }
        if (!ok) {
            record_status(LA_ERR_BAD_SEQLENS);
            continue;
        }
        out[i] = acc;
    }
}

}  // namespace la
