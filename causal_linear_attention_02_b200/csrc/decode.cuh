// Recurrent decode step: S <- S + k^T v ; o = q S  (O(d^2) per token; page
// "MiniMax-01 Lightning Attention", sections "Lightning Attention 设计" and
// "与标准 Softmax Attention 的区别": inference only updates the d x d KV state).
//
// Bandwidth-bound: each (sequence, head) reads and writes its d x d fp32 state
// once. The output is formed from the OLD state while it streams through
// registers, o = q S_old + (q . k) v, so the new state is written once and never
// re-read. One CTA per (sequence, head): a warp covers whole rows with 16-byte
// coalesced streaming loads/stores; the partial outputs of the row groups are
// reduced through shared memory.
//
// The kDecay instance takes a per-head decay rate (decay.cuh):
// S <- lambda_h S + k^T v, o = lambda_h (q S_old) + (q . k) v.
#pragma once

#include "common.cuh"
#include "decay.cuh"

namespace la {

// Threads per CTA: CG float4 column groups times RG row groups, RG the largest
// divisor of D with CG * RG <= 256.
__host__ __device__ constexpr int decode_row_groups(int D) {
    int best = 1;
    for (int r = 1; r <= D; ++r)
        if (D % r == 0 && (D / 4) * r <= 256) best = r;
    return best;
}

template <typename Tin, int D, bool kDecay = false>
__global__ void __launch_bounds__((D / 4) * decode_row_groups(D))
decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                   float* __restrict__ state, Tin* __restrict__ o, const float* decay, int H) {
    constexpr int CG = D / 4;                 // float4 column groups per row
    constexpr int RG = decode_row_groups(D);  // row groups (threads sharing a column group)
    constexpr int NT = CG * RG;
    constexpr int ROWS = D / RG;              // rows per thread
    static_assert(D % 4 == 0 && NT >= D, "decode tiling");
    __shared__ float qs[D], ks[D], vs[D];
    __shared__ float4 red[RG][CG];
    const int64_t p = blockIdx.x;             // (sequence, head) pair
    const int tid = threadIdx.x;
    float lam = 1.f;
    if constexpr (kDecay) {
        lam = decay[p % H];
        if (!(lam >= 0.f && lam <= 1.f)) {
            if (tid == 0) record_status(LA_ERR_BAD_DECAY);
            return;
        }
    }
    if (tid < D) {
        qs[tid] = io<Tin>::ld(q + p * D + tid);
        ks[tid] = io<Tin>::ld(k + p * D + tid);
        vs[tid] = io<Tin>::ld(v + p * D + tid);
    }
    const int cg = tid % CG, rg = tid / CG;
    float4* S = reinterpret_cast<float4*>(state + p * D * D);
    float4 rows[ROWS];
#pragma unroll
    for (int a = 0; a < ROWS; ++a) rows[a] = __ldcs(S + (int64_t)(rg + a * RG) * CG + cg);
    __syncthreads();
    const float4 vv = make_float4(vs[4 * cg], vs[4 * cg + 1], vs[4 * cg + 2], vs[4 * cg + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int a = 0; a < ROWS; ++a) {
        const int i = rg + a * RG;
        const float qi = qs[i], ki = ks[i];
        float4 s = rows[a];
        acc.x = fmaf(qi, s.x, acc.x); acc.y = fmaf(qi, s.y, acc.y);
        acc.z = fmaf(qi, s.z, acc.z); acc.w = fmaf(qi, s.w, acc.w);
        if constexpr (kDecay) {
            s.x = fmaf(ki, vv.x, lam * s.x); s.y = fmaf(ki, vv.y, lam * s.y);
            s.z = fmaf(ki, vv.z, lam * s.z); s.w = fmaf(ki, vv.w, lam * s.w);
        } else {
            s.x = fmaf(ki, vv.x, s.x); s.y = fmaf(ki, vv.y, s.y);
            s.z = fmaf(ki, vv.z, s.z); s.w = fmaf(ki, vv.w, s.w);
        }
        __stcs(S + (int64_t)i * CG + cg, s);
    }
    red[rg][cg] = acc;
    __syncthreads();
    if (tid < D) {
        float qk = 0.f;                       // q . k for the current token's own term
        for (int x = 0; x < D; ++x) qk = fmaf(qs[x], ks[x], qk);
        const int c = tid / 4, lane4 = tid % 4;
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            const float4 x = red[r][c];
            sum += lane4 == 0 ? x.x : lane4 == 1 ? x.y : lane4 == 2 ? x.z : x.w;
        }
        if constexpr (kDecay) sum *= lam;
        io<Tin>::st(o + p * D + tid, fmaf(qk, vs[tid], sum));
    }
}

}  // namespace la
