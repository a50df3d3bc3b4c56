// Tensor-core (tcgen05 + TMEM + TMA) kernels for bf16 prefill with d = 128.
//
// The method (page "MiniMax-01 Lightning Attention", section "Lightning
// Attention 设计"; page "首个线性注意力架构的大模型来了…", section "4.1 创新的线性
// 注意力"): inside a block of B tokens the left product (Q_b K_b^T, causal
// mask) V_b; across blocks the right product Q_b . KV_prefix(b), where
// KV_prefix(b) = S0 + sum_{c<b} K_c^T V_c.
//
// Work unit of the prefill kernel: 128 query rows ("half" r of a B = 256 block,
// or the whole block when B = 128) of one head. Its keys are streamed in
// 64-token chunks j = 0 .. 2r+1 through a ring of shared-memory stages:
//   S_j  = Q K_j^T                 tcgen05, M=128 N=64  K=128, A,B K-major, D in TMEM
//   P_j  = mask(S_j) -> bf16       4 warps: TMEM -> registers -> TMEM (in place)
//   O   += P_j V_j                 tcgen05, M=128 N=128 K=64,  A from TMEM, B MN-major
// then  O += Q . prefix            tcgen05, M=128 N=128 K=128, B MN-major (bf16 prefix)
// and the 4 warps convert O to bf16 and store it.
//
// Shared-memory operand tiles are written by TMA with 128-byte swizzle and
// read by the MMA through SWIZZLE_128B descriptors: a 64-element (128 B) row
// per token, 8-row (1024 B) swizzle atoms.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace la {
namespace tc {

using namespace la::sm100;

constexpr int D = 128;            // head dim served by this path
constexpr int UM = 128;           // query rows per work unit (MMA M)
constexpr int KC = 64;            // keys per streamed chunk
constexpr int NKV = 3;            // K/V ring stages

constexpr uint32_t Q_BYTES = UM * D * 2;           // 32 KB (two 16 KB d-halves)
constexpr uint32_t QH_BYTES = UM * 64 * 2;         // 16 KB: one 64-column half of Q
constexpr uint32_t KV_BYTES = KC * D * 2;          // 16 KB per K or V chunk
constexpr uint32_t KVH_BYTES = KC * 64 * 2;        // 8 KB: one 64-column half of a chunk
constexpr uint32_t PRE_BYTES = D * D * 2;          // 32 KB bf16 prefix
constexpr uint32_t PREH_BYTES = D * 64 * 2;        // 16 KB: one 64-column half

// shared memory map of the prefill kernel (offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;                                   // 2 stages
constexpr uint32_t OFF_KV = OFF_Q + 2 * Q_BYTES;                // NKV stages of (K, V)
constexpr uint32_t OFF_PRE = OFF_KV + NKV * 2 * KV_BYTES;
constexpr uint32_t OFF_BAR = OFF_PRE + PRE_BYTES;
constexpr uint32_t SMEM_PREFILL = OFF_BAR + 1024 + 1024;        // barriers + alignment slack

// TMEM columns (fp32 accumulators, 128 lanes)
constexpr uint32_t TM_O = 0;        // two 128-column O accumulators
constexpr uint32_t TM_S = 256;      // two 64-column score buffers (P written over their first 32)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_S = idesc_bf16(128, 64, false, false);    // Q K^T
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, false, true);   // P V (A from TMEM)
constexpr uint32_t IDESC_QP = idesc_bf16(128, 128, false, true);   // Q prefix
constexpr uint32_t IDESC_KV = idesc_bf16(128, 128, true, true);    // K^T V

struct Bars {
    uint64_t q_full[2], q_empty[2];
    uint64_t kv_full[NKV], kv_empty[NKV];
    uint64_t pre_full, pre_empty;
    uint64_t s_full[2], p_full[2];
    uint64_t o_full[2], o_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};

struct Unit {
    int g, r, h;
    BlockEntry e;
    int rows;   // valid query rows of this unit (<= 0: nothing to do)
    int nkc;    // key chunks to stream
};

__device__ __forceinline__ Unit decode_unit(int64_t u, int H, int R, const BlockEntry* table) {
    Unit x;
    x.h = (int)(u % H);
    x.r = (int)((u / H) % R);
    x.g = (int)(u / ((int64_t)H * R));
    x.e = table[x.g];
    x.rows = min(UM, x.e.len - UM * x.r);
    const int kmax = (x.r + 1) * (UM / KC);                       // chunks up to the diagonal
    x.nkc = min(kmax, (x.e.len + KC - 1) / KC);
    return x;
}

// ----------------------------------------------------------------------------
// Prefill kernel. 192 threads: warp 0 TMA producer, warp 1 MMA issuer (and
// TMEM owner), warps 2..5 score->P conversion and O epilogue. Persistent:
// CTA c takes units c, c + gridDim.x, ... in increasing order.
// prefix: bf16 [block][H][D][D] read through tmP (2D: {D, rows}).
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(192, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmP,
                  __nv_bfloat16* __restrict__ out, const BlockEntry* __restrict__ table,
                  const Control* __restrict__ ctrl, int H, int R, uint64_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort_flag = &bars->abort_flag;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->q_full[i], 1);  mbar_init(&bars->q_empty[i], 1);
            mbar_init(&bars->s_full[i], 1);  mbar_init(&bars->p_full[i], 128);
            mbar_init(&bars->o_full[i], 1);  mbar_init(&bars->o_empty[i], 128);
        }
        for (int i = 0; i < NKV; ++i) { mbar_init(&bars->kv_full[i], 1); mbar_init(&bars->kv_empty[i], 1); }
        mbar_init(&bars->pre_full, 1);
        mbar_init(&bars->pre_empty, 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmP);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const int64_t nunits = ctrl->ok ? (int64_t)ctrl->nblocks * R * H : 0;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0, kv_it = 0;
            for (int64_t u = blockIdx.x; u < nunits; u += gridDim.x) {
                const Unit x = decode_unit(u, H, R, table);
                if (x.rows <= 0) continue;
                const int tq = x.e.tok0 + UM * x.r;
                const uint32_t qs = it & 1;
                if (!mbar_wait(&bars->q_empty[qs], ((it >> 1) & 1) ^ 1, abort_flag, wait_ns)) break;
                uint8_t* qdst = smem + OFF_Q + qs * Q_BYTES;
                mbar_expect_tx(&bars->q_full[qs], Q_BYTES);
                tma_load_3d(qdst, &tmQ, &bars->q_full[qs], 0, x.h, tq);
                tma_load_3d(qdst + QH_BYTES, &tmQ, &bars->q_full[qs], 64, x.h, tq);
                bool ok = true;
                for (int j = 0; j < x.nkc; ++j, ++kv_it) {
                    const uint32_t st = kv_it % NKV;
                    if (!mbar_wait(&bars->kv_empty[st], ((kv_it / NKV) & 1) ^ 1, abort_flag, wait_ns)) { ok = false; break; }
                    uint8_t* kdst = smem + OFF_KV + st * 2 * KV_BYTES;
                    uint8_t* vdst = kdst + KV_BYTES;
                    const int tk = x.e.tok0 + KC * j;
                    mbar_expect_tx(&bars->kv_full[st], 2 * KV_BYTES);
                    tma_load_3d(kdst, &tmK, &bars->kv_full[st], 0, x.h, tk);
                    tma_load_3d(kdst + KVH_BYTES, &tmK, &bars->kv_full[st], 64, x.h, tk);
                    tma_load_3d(vdst, &tmV, &bars->kv_full[st], 0, x.h, tk);
                    tma_load_3d(vdst + KVH_BYTES, &tmV, &bars->kv_full[st], 64, x.h, tk);
                }
                if (!ok) break;
                if (!mbar_wait(&bars->pre_empty, (it & 1) ^ 1, abort_flag, wait_ns)) break;
                const int prow = (x.g * H + x.h) * D;
                mbar_expect_tx(&bars->pre_full, PRE_BYTES);
                tma_load_2d(smem + OFF_PRE, &tmP, &bars->pre_full, 0, prow);
                tma_load_2d(smem + OFF_PRE + PREH_BYTES, &tmP, &bars->pre_full, 64, prow);
                ++it;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, kv_it = 0, s_it = 0;
            const uint32_t q_base = smem_u32(smem + OFF_Q);
            const uint32_t kv_base = smem_u32(smem + OFF_KV);
            const uint32_t pre_base = smem_u32(smem + OFF_PRE);
            for (int64_t u = blockIdx.x; u < nunits; u += gridDim.x) {
                const Unit x = decode_unit(u, H, R, table);
                if (x.rows <= 0) continue;
                const uint32_t qs = it & 1, ob = it & 1;
                if (!mbar_wait(&bars->q_full[qs], (it >> 1) & 1, abort_flag, wait_ns)) break;
                if (!mbar_wait(&bars->o_empty[ob], ((it >> 1) & 1) ^ 1, abort_flag, wait_ns)) break;
                tc_fence_after();
                const uint32_t qa = q_base + qs * Q_BYTES;
                const uint32_t d_o = tmem + TM_O + ob * 128;
                bool ok = true;
                // S_j = Q K_j^T into score buffer (s_it + j) & 1
                auto issue_scores = [&](int j) -> bool {
                    const uint32_t kvi = kv_it + j;
                    const uint32_t st = kvi % NKV;
                    if (!mbar_wait(&bars->kv_full[st], (kvi / NKV) & 1, abort_flag, wait_ns)) return false;
                    tc_fence_after();
                    const uint32_t kb = kv_base + st * 2 * KV_BYTES;
                    const uint32_t d_s = tmem + TM_S + ((s_it + j) & 1) * 64;
#pragma unroll
                    for (int s = 0; s < D / 16; ++s) {
                        const uint32_t koff = (s >> 2) * QH_BYTES + (s & 3) * 32;
                        const uint32_t kkoff = (s >> 2) * KVH_BYTES + (s & 3) * 32;
                        mma_ss(d_s, sdesc_sw128(qa + koff, 16, 1024), sdesc_sw128(kb + kkoff, 16, 1024),
                               IDESC_S, s > 0);
                    }
                    tc_commit(&bars->s_full[(s_it + j) & 1]);
                    return true;
                };
                if (!issue_scores(0)) break;
                for (int j = 0; j < x.nkc; ++j) {
                    if (j + 1 < x.nkc && !issue_scores(j + 1)) { ok = false; break; }
                    const uint32_t sb = (s_it + j) & 1;
                    if (!mbar_wait(&bars->p_full[sb], ((s_it + j) >> 1) & 1, abort_flag, wait_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = (kv_it + j) % NKV;
                    const uint32_t vb = kv_base + st * 2 * KV_BYTES + KV_BYTES;
                    const uint32_t a_p = tmem + TM_S + sb * 64;
#pragma unroll
                    for (int s = 0; s < KC / 16; ++s) {
                        // A: 16 keys of P = 8 TMEM columns; B: 16 rows (tokens) of V = 2 swizzle atoms
                        mma_ts(d_o, a_p + s * 8, sdesc_sw128(vb + s * 2048, KVH_BYTES, 1024), IDESC_PV,
                               (j > 0 || s > 0));
                    }
                    tc_commit(&bars->kv_empty[st]);
                }
                if (!ok) break;
                kv_it += x.nkc;
                s_it += x.nkc;
                // inter-block right product with the prefix state
                if (!mbar_wait(&bars->pre_full, it & 1, abort_flag, wait_ns)) break;
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < D / 16; ++s) {
                    const uint32_t koff = (s >> 2) * QH_BYTES + (s & 3) * 32;
                    mma_ss(d_o, sdesc_sw128(qa + koff, 16, 1024),
                           sdesc_sw128(pre_base + s * 2048, PREH_BYTES, 1024), IDESC_QP, 1);
                }
                tc_commit(&bars->pre_empty);
                tc_commit(&bars->q_empty[qs]);
                tc_commit(&bars->o_full[ob]);
                ++it;
            }
        }
    } else {
        // ------------------------------------------------------------ P conversion + epilogue
        const int quad = warp & 3;                       // TMEM lane quadrant of this warp
        const int m = quad * 32 + lane;                  // row of the unit owned by this thread
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        uint32_t it = 0, s_it = 0;
        for (int64_t u = blockIdx.x; u < nunits; u += gridDim.x) {
            const Unit x = decode_unit(u, H, R, table);
            if (x.rows <= 0) continue;
            bool ok = true;
            const int qi = UM * x.r + m;                 // query position inside the block
            for (int j = 0; j < x.nkc; ++j, ++s_it) {
                const uint32_t sb = s_it & 1;
                if (!mbar_wait(&bars->s_full[sb], (s_it >> 1) & 1, abort_flag, wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ts = tmem + lane_base + TM_S + sb * 64;
                uint32_t a[32], b[32];
                tmem_ld_x32(ts, a);
                tmem_ld_x32(ts + 32, b);
                tmem_wait_ld();
                const int lim = qi - KC * j;             // keep key column c when c <= lim
                uint32_t p[32];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float s0 = __uint_as_float(a[2 * c]), s1 = __uint_as_float(a[2 * c + 1]);
                    p[c] = pack_bf16x2(2 * c <= lim ? s0 : 0.f, 2 * c + 1 <= lim ? s1 : 0.f);
                }
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float s0 = __uint_as_float(b[2 * c]), s1 = __uint_as_float(b[2 * c + 1]);
                    p[16 + c] = pack_bf16x2(32 + 2 * c <= lim ? s0 : 0.f, 33 + 2 * c <= lim ? s1 : 0.f);
                }
                tmem_st_x32(ts, p);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[sb]);
            }
            if (!ok) break;
            const uint32_t ob = it & 1;
            if (!mbar_wait(&bars->o_full[ob], (it >> 1) & 1, abort_flag, wait_ns)) break;
            tc_fence_after();
            const bool valid = m < x.rows;
            __nv_bfloat16* orow = out + ((int64_t)(x.e.tok0 + UM * x.r + m) * H + x.h) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t r[32];
                tmem_ld_x32(tmem + lane_base + TM_O + ob * 128 + c0, r);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint4 pk;
                        pk.x = pack_bf16x2(__uint_as_float(r[8 * w + 0]), __uint_as_float(r[8 * w + 1]));
                        pk.y = pack_bf16x2(__uint_as_float(r[8 * w + 2]), __uint_as_float(r[8 * w + 3]));
                        pk.z = pack_bf16x2(__uint_as_float(r[8 * w + 4]), __uint_as_float(r[8 * w + 5]));
                        pk.w = pack_bf16x2(__uint_as_float(r[8 * w + 6]), __uint_as_float(r[8 * w + 7]));
                        *reinterpret_cast<uint4*>(orow + c0 + 8 * w) = pk;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->o_empty[ob]);
            ++it;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ----------------------------------------------------------------------------
// Block-state kernel: U[g][h] = K_g^T V_g (fp32) for every full block, on the
// tensor cores. One CTA (128 threads) per (block, head); the whole block is
// loaded by TMA, then 4 x (B/64) MMAs of M=128 (key dim i) N=128 (value dim j)
// K=16 (tokens) accumulate into TMEM, with both operands MN-major (the token
// rows staged by TMA are the K dimension of this product). Partial (last)
// blocks are skipped: a prefill never needs their state.
// ----------------------------------------------------------------------------
constexpr uint32_t SMEM_STATE_MAX = 2 * 256 * D * 2 + 1024 + 256;

__global__ void __launch_bounds__(128, 1)
block_state_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      float* __restrict__ U, const BlockEntry* __restrict__ table,
                      const Control* __restrict__ ctrl, int H, int B, uint64_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t kv_bytes = (uint32_t)B * D * 2;
    uint8_t* ks = smem;
    uint8_t* vs = smem + kv_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * kv_bytes);
    uint64_t* done = full + 1;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int64_t g = blockIdx.x / H;
    const int h = blockIdx.x % H;
    if (!ctrl->ok || g >= ctrl->nblocks) return;
    const BlockEntry e = table[g];
    if (e.len != B) return;

    if (threadIdx.x == 0) {
        mbar_init(full, 1);
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(tslot, 128); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const int nch = B / KC;

    if (threadIdx.x == 0) {
        mbar_expect_tx(full, 2 * kv_bytes);
        for (int c = 0; c < nch; ++c) {
            const int t = e.tok0 + KC * c;
            tma_load_3d(ks + c * KV_BYTES, &tmK, full, 0, h, t);
            tma_load_3d(ks + c * KV_BYTES + KVH_BYTES, &tmK, full, 64, h, t);
            tma_load_3d(vs + c * KV_BYTES, &tmV, full, 0, h, t);
            tma_load_3d(vs + c * KV_BYTES + KVH_BYTES, &tmV, full, 64, h, t);
        }
        if (mbar_wait(full, 0, abort_flag, wait_ns)) {
            tc_fence_after();
            const uint32_t ka = smem_u32(ks), vb = smem_u32(vs);
            for (int c = 0; c < nch; ++c) {
#pragma unroll
                for (int s = 0; s < KC / 16; ++s) {
                    const uint32_t off = c * KV_BYTES + s * 2048;
                    mma_ss(tmem, sdesc_sw128(ka + off, KVH_BYTES, 1024), sdesc_sw128(vb + off, KVH_BYTES, 1024),
                           IDESC_KV, (c > 0 || s > 0));
                }
            }
            tc_commit(done);
        }
    }
    __syncwarp();
    if (mbar_wait(done, 0, abort_flag, wait_ns)) {
        tc_fence_after();
        const int i = warp * 32 + lane;                   // row of U (key dim) = TMEM lane
        float* urow = U + (((int64_t)g * H + h) * D + i) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t r[32];
            tmem_ld_x32(tmem + (uint32_t(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int w = 0; w < 8; ++w)
                *reinterpret_cast<float4*>(urow + c0 + 4 * w) =
                    make_float4(__uint_as_float(r[4 * w]), __uint_as_float(r[4 * w + 1]),
                                __uint_as_float(r[4 * w + 2]), __uint_as_float(r[4 * w + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

}  // namespace tc
}  // namespace la
