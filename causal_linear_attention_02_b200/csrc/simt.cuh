// CUDA-core (SIMT) prefill kernels for the shapes the tensor-core path does
// not cover: fp32 inputs (computed in fp32 end to end), head dims other than
// 128 and block size 64. Same decomposition as the tensor-core path
// (page "MiniMax-01 Lightning Attention", section "Lightning Attention 设计"):
//   block_state_simt : U_b = K_b^T V_b over the valid rows of block b
//   (chain_scan_kernel turns U into per-block prefix states)
//   prefill_simt     : O_b = (Q_b K_b^T masked) V_b + Q_b . prefix_b
// The kDecay instances add a per-head decay rate on the state (decay.cuh): key
// rows weighted lambda^(n-1-r) in U_b, the decay mask lambda^(t-u) on the
// scores and lambda^(r+1) on the inter-block product.
#pragma once

#include "common.cuh"
#include "decay.cuh"

namespace la {
namespace simt {

constexpr int THREADS = 256;

// U[g][h] = sum over the valid tokens t of block g of k_t^T v_t (fp32).
// One CTA per (block, head); tokens staged through shared memory 32 at a time.
// Thread (ti, tj) of a 16 x 16 grid owns the (D/16) x (D/16) micro-tile
// rows ti*(D/16).., cols tj*(D/16)...
template <typename Tin, int D, bool kDecay = false>
__global__ void __launch_bounds__(THREADS) block_state_simt(const Tin* __restrict__ k, const Tin* __restrict__ v,
                                                            const BlockEntry* __restrict__ table,
                                                            const Control* __restrict__ ctrl, int H,
                                                            float* __restrict__ U, const float* decay) {
    constexpr int MT = D / 16;
    constexpr int CH = 32;
    __shared__ float ks[CH][D];
    __shared__ float vs[CH][D];
    const int64_t g = blockIdx.x / H;
    const int h = blockIdx.x % H;
    if (g >= ctrl->nblocks) return;
    const BlockEntry e = table[g];
    float l2 = 0.f;
    if constexpr (kDecay) {
        if (!load_decay(decay, h, l2)) return;
    }
    const int tid = threadIdx.x, ti = tid / 16, tj = tid % 16;
    float acc[MT][MT];
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b = 0; b < MT; ++b) acc[a][b] = 0.f;
    for (int t0 = 0; t0 < e.len; t0 += CH) {
        const int n = min(CH, e.len - t0);
        for (int x = tid; x < CH * D; x += THREADS) {
            const int r = x / D, c = x % D;
            float kv = 0.f, vv = 0.f;
            if (r < n) {
                const int64_t off = ((int64_t)(e.tok0 + t0 + r) * H + h) * D + c;
                kv = io<Tin>::ld(k + off);
                vv = io<Tin>::ld(v + off);
                if constexpr (kDecay) kv *= decay_pow(l2, e.len - 1 - (t0 + r));
            }
            ks[r][c] = kv;
            vs[r][c] = vv;
        }
        __syncthreads();
        for (int r = 0; r < n; ++r) {
            float kr[MT], vr[MT];
#pragma unroll
            for (int a = 0; a < MT; ++a) kr[a] = ks[r][ti * MT + a];
#pragma unroll
            for (int b = 0; b < MT; ++b) vr[b] = vs[r][tj * MT + b];
#pragma unroll
            for (int a = 0; a < MT; ++a)
#pragma unroll
                for (int b = 0; b < MT; ++b) acc[a][b] = fmaf(kr[a], vr[b], acc[a][b]);
        }
        __syncthreads();
    }
    float* u = U + ((int64_t)g * H + h) * D * D;
#pragma unroll
    for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b = 0; b < MT; ++b) u[(ti * MT + a) * D + tj * MT + b] = acc[a][b];
}

// O for one 64-row query tile of one block of one head.
//   acc  = Q_tile . prefix_g                        (inter-block right product)
//   acc += sum over 64-key tiles kt <= qt of (Q_tile K_kt^T masked) V_kt  (intra left product)
// prefix is fp32 [block][H][D][D]. Thread (ti, tj) of 16 x 16 owns rows
// ti*4..ti*4+3 and columns tj*(D/16)...
template <typename Tin, int D, bool kDecay = false>
__global__ void __launch_bounds__(THREADS) prefill_simt(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                        const Tin* __restrict__ v, Tin* __restrict__ o,
                                                        const float* __restrict__ prefix,
                                                        const BlockEntry* __restrict__ table,
                                                        const Control* __restrict__ ctrl, int H, int B,
                                                        const float* decay) {
    constexpr int MT = D / 16;
    constexpr int QT = 64;
    extern __shared__ float4 smem_f4[];
    float* smem = reinterpret_cast<float*>(smem_f4);
    float* qs = smem;                 // [QT][D]
    float* ks = qs + QT * D;          // [QT][D]  (also prefix rows)
    float* vs = ks + QT * D;          // [QT][D]
    float* ss = vs + QT * D;          // [QT][QT + 1]
    const int tiles = B / QT;
    const int64_t g = blockIdx.x / (H * tiles);
    const int rem = blockIdx.x % (H * tiles);
    const int qt = rem / H, h = rem % H;
    if (g >= ctrl->nblocks) return;
    const BlockEntry e = table[g];
    const int r0 = qt * QT;
    if (r0 >= e.len) return;
    const int nq = min(QT, e.len - r0);
    float l2 = 0.f;
    if constexpr (kDecay) {
        if (!load_decay(decay, h, l2)) return;
    }
    const int tid = threadIdx.x, ti = tid / 16, tj = tid % 16;

    for (int x = tid; x < QT * D; x += THREADS) {
        const int r = x / D, c = x % D;
        qs[x] = r < nq ? io<Tin>::ld(q + ((int64_t)(e.tok0 + r0 + r) * H + h) * D + c) : 0.f;
    }
    float acc[4][MT];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < MT; ++b) acc[a][b] = 0.f;

    // inter-block: Q . prefix, prefix rows staged QT at a time through ks
    const float* pre = prefix + ((int64_t)g * H + h) * D * D;
    for (int i0 = 0; i0 < D; i0 += QT) {
        const int ni = min(QT, D - i0);
        __syncthreads();
        for (int x = tid; x < ni * D; x += THREADS) ks[x] = pre[(int64_t)i0 * D + x];
        __syncthreads();
        for (int i = 0; i < ni; ++i) {
            float pr[MT];
#pragma unroll
            for (int b = 0; b < MT; ++b) pr[b] = ks[i * D + tj * MT + b];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float qa = qs[(ti * 4 + a) * D + i0 + i];
#pragma unroll
                for (int b = 0; b < MT; ++b) acc[a][b] = fmaf(qa, pr[b], acc[a][b]);
            }
        }
    }
    if constexpr (kDecay) {   // lambda^(r+1) on the inter-block product of row r of the block
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const float w = decay_pow(l2, r0 + ti * 4 + a + 1);
#pragma unroll
            for (int b = 0; b < MT; ++b) acc[a][b] *= w;
        }
    }
    // intra-block: key tiles up to and including the diagonal tile
    for (int kt = 0; kt <= qt; ++kt) {
        const int k0 = kt * QT;
        const int nk = min(QT, e.len - k0);
        __syncthreads();
        for (int x = tid; x < QT * D; x += THREADS) {
            const int r = x / D, c = x % D;
            float kv = 0.f, vv = 0.f;
            if (r < nk) {
                const int64_t off = ((int64_t)(e.tok0 + k0 + r) * H + h) * D + c;
                kv = io<Tin>::ld(k + off);
                vv = io<Tin>::ld(v + off);
            }
            ks[x] = kv;
            vs[x] = vv;
        }
        __syncthreads();
        // scores: thread (ti, tj) -> rows ti*4.., keys tj*4..
        {
            float sc[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) sc[a][b] = 0.f;
            for (int c = 0; c < D; ++c) {
                float qa[4], kb[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) qa[a] = qs[(ti * 4 + a) * D + c];
#pragma unroll
                for (int b = 0; b < 4; ++b) kb[b] = ks[(tj * 4 + b) * D + c];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) sc[a][b] = fmaf(qa[a], kb[b], sc[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int qi = r0 + ti * 4 + a, kj = k0 + tj * 4 + b;   // positions in the block
                    float x = (kj <= qi && kj < e.len) ? sc[a][b] : 0.f;
                    if constexpr (kDecay) x *= decay_pow(l2, max(qi - kj, 0));
                    ss[(ti * 4 + a) * (QT + 1) + tj * 4 + b] = x;
                }
        }
        __syncthreads();
        for (int j = 0; j < nk; ++j) {
            float vb[MT];
#pragma unroll
            for (int b = 0; b < MT; ++b) vb[b] = vs[j * D + tj * MT + b];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float sa = ss[(ti * 4 + a) * (QT + 1) + j];
#pragma unroll
                for (int b = 0; b < MT; ++b) acc[a][b] = fmaf(sa, vb[b], acc[a][b]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int r = ti * 4 + a;
        if (r < nq) {
            Tin* orow = o + ((int64_t)(e.tok0 + r0 + r) * H + h) * D;
#pragma unroll
            for (int b = 0; b < MT; ++b) io<Tin>::st(orow + tj * MT + b, acc[a][b]);
        }
    }
}

template <int D>
constexpr size_t prefill_simt_smem() {
    return (size_t)(3 * 64 * D + 64 * 65) * sizeof(float);
}

}  // namespace simt
}  // namespace la
