// Helpers of the prefill's backward pass (the training pass; the pages give the
// forward only). With S_t = S0 + sum_{s <= t} k_s^T v_s and L = sum_t dO_t . O_t:
//   dQ_t = dO_t S_t^T                    -> a forward prefill of (dO, V, K) from S0^T
//   dV_s = sum_{t >= s} (k_s . q_t) dO_t -> an anti-causal prefill of (K, Q, dO)
//   dK_s = sum_{t >= s} (dO_t . v_s) q_t -> an anti-causal prefill of (V, dO, Q)
//   dS0  = sum_t q_t^T dO_t              -> the state of (Q, dO)
// so the pass reuses the forward kernels. The on-chip-state kernel has an
// anti-causal instance; on the other paths (and with decay) the anti-causal
// prefills are causal prefills over every sequence reversed, reversed back.
// These kernels reverse the token order inside every sequence (that path) and
// transpose the carried-in states.
#pragma once

#include "common.cuh"

namespace la {

// out[start + end - 1 - t] = in[t] for every token t of every sequence [start, end),
// one 16-byte group per thread and iteration (rows of `row16` groups). A
// sequence whose bounds are not inside [0, T] is skipped and reported as
// LA_ERR_BAD_SEQLENS (the prefills that follow report it too).
__global__ void __launch_bounds__(256)
reverse_tokens_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, const int32_t* cu, int nseq,
                      int64_t T, int64_t row16) {
    for (int s = blockIdx.y; s < nseq; s += gridDim.y) {
        const int64_t start = cu ? cu[s] : 0, end = cu ? cu[s + 1] : T;
        if (start < 0 || end > T || start > end) {
            if (blockIdx.x == 0 && threadIdx.x == 0) record_status(LA_ERR_BAD_SEQLENS);
            continue;
        }
        const int64_t n = (end - start) * row16;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
            const int64_t t = start + i / row16, c = i % row16;
            out[(start + end - 1 - t) * row16 + c] = __ldcs(in + t * row16 + c);
        }
    }
}

// out[p][j][i] = in[p][i][j] for p < n, d x d fp32 matrices, through a 32 x 33
// shared tile (blockIdx.x: matrix p; y, z: the tile).
__global__ void __launch_bounds__(256)
transpose_states_kernel(const float* __restrict__ in, float* __restrict__ out, int d) {
    __shared__ float tile[32][33];
    const int64_t base = (int64_t)blockIdx.x * d * d;
    const int i0 = blockIdx.y * 32, j0 = blockIdx.z * 32;
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int i = i0 + r, j = j0 + threadIdx.x;
        if (i < d && j < d) tile[r][threadIdx.x] = in[base + (int64_t)i * d + j];
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int j = j0 + r, i = i0 + threadIdx.x;
        if (i < d && j < d) out[base + (int64_t)j * d + i] = tile[threadIdx.x][r];
    }
}

// states[i] *= lambda_h for every (sequence, head) state of [nseq][H][d][d]
// (the decay variant's dS0 = lambda R_start); float4 groups, grid-stride.
__global__ void __launch_bounds__(256)
scale_states_kernel(float4* states, const float* decay, int H, int64_t per_state4, int64_t total4) {
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total4; i += step) {
        const float lam = decay[(i / per_state4) % H];
        float4 x = states[i];
        x.x *= lam; x.y *= lam; x.z *= lam; x.w *= lam;
        states[i] = x;
    }
}

}  // namespace la
