// Final recurrent state of each sequence on the tensor cores: bf16, d = 128.
//
//   state[s][h] = S0[s][h] + sum_{t in seq s} k_t^T v_t
//
// (the d x d KV state that the right product carries from block to block and
// the decode step continues from; page "MiniMax-01 Lightning Attention",
// section "Lightning Attention 设计"). Column j of the state depends on column
// j of V only, so one (sequence, head) splits into two halves of 64 value
// columns; each half is a work item, taken round-robin by persistent CTAs.
// A work item streams its keys in chunks of 128 and accumulates
// K_c^T V_c (M=128, N=64, K=128) into a fp32 TMEM accumulator; the rows of the
// last chunk that lie past the sequence end are zeroed in shared memory first
// (they belong to the next sequence). Roles (256 threads):
//   warp 0 (lane 0)  TMA producer of K and V chunks (4 stages of 48 KB)
//   warp 1 (lane 0)  tcgen05 issuer; two accumulators, so one work item's
//                    result can be read out while the next accumulates
//   warp 2           zeroes the tail rows of a partial last chunk when the
//                    issuer hands it over (one request / done pair per chunk)
//   warps 4-7        read the accumulator, add S0, store the state rows
// Every wait is bounded; on expiry the CTA records LA_ERR_TIMEOUT and exits.
#pragma once

#include "common.cuh"
#include "sm100.cuh"
#include "pipe.cuh"

namespace la {
namespace state {

using namespace la::sm100;

constexpr int D = 128, DV = 64, KC = 128;
constexpr int NKV = 4;
constexpr int NTHREADS = 256;
constexpr uint32_t KH_BYTES = KC * 64 * 2;           // 16 KB
constexpr uint32_t K_BYTES = 2 * KH_BYTES;           // 32 KB
constexpr uint32_t V_BYTES = KC * DV * 2;            // 16 KB
constexpr uint32_t STAGE = K_BYTES + V_BYTES;        // 48 KB
constexpr uint32_t OFF_BAR = NKV * STAGE;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
constexpr uint32_t TM_COLS = 128;                    // two accumulators of 64 columns
constexpr uint32_t IDESC_KV = idesc_bf16(D, DV, true, true);   // K^T (MN-major) x V (MN-major)

struct Bars {
    uint64_t full[NKV], empty[NKV];
    uint64_t fix_req, fix_done;   // issuer <-> warp 2, once per partial last chunk, in order
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct Params {
    float* out;               // [nseq][H][D][D]
    const float* init;        // [nseq][H][D][D] or nullptr
    const SeqEntry* seqs;
    const Control* ctrl;
    int H, nseq;
    uint64_t wait_ns;
};

// Work items w = 2 * (seq * H + head) + half, round-robin over the CTAs.
struct Item {
    int64_t w, nitems;
    int step, seq, h, half, tok0, len, nch;
    uint32_t kc0, a;          // first chunk (ring index) and accumulator count of this item
    bool valid;
    __device__ __forceinline__ void load(const Params& p) {
        valid = w < nitems;
        if (!valid) return;
        const int64_t pair = w >> 1;
        seq = (int)(pair / p.H);
        h = (int)(pair % p.H);
        half = (int)(w & 1);
        const SeqEntry e = p.seqs[seq];
        tok0 = e.tok0;
        len = e.len;
        nch = (len + KC - 1) / KC;
    }
    __device__ __forceinline__ void init(const Params& p) {
        w = blockIdx.x;
        step = gridDim.x;
        nitems = p.ctrl->ok ? (int64_t)p.nseq * p.H * 2 : 0;
        kc0 = 0;
        a = 0;
        load(p);
    }
    __device__ __forceinline__ void next(const Params& p) {
        kc0 += nch;
        if (nch > 0) ++a;
        w += step;
        load(p);
    }
};

__global__ void __launch_bounds__(NTHREADS, 1)
state_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&bars->abort_flag, const_cast<volatile int*>(&p.ctrl->abort), p.wait_ns};

    if (threadIdx.x == 0) {
        for (int i = 0; i < NKV; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], 1);
        }
        mbar_init(&bars->fix_req, 1);
        mbar_init(&bars->fix_done, 32);
        for (int i = 0; i < 2; ++i) { mbar_init(&bars->acc_full[i], 1); mbar_init(&bars->acc_empty[i], 128); }
        mbar_init(&bars->drain, 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            const uint64_t once = policy_evict_first();
            Item it;
            it.init(p);
            uint32_t issued = 0;
            bool ok = true;
            while (ok && it.valid) {
                for (int c = 0; c < it.nch; ++c) {
                    const uint32_t kc = it.kc0 + c, st = kc % NKV;
                    if (!wait_bar(&bars->empty[st], ((kc / NKV) & 1) ^ 1, ab)) { ok = false; break; }
                    uint8_t* d = smem + st * STAGE;
                    const int t = it.tok0 + KC * c;
                    mbar_expect_tx(&bars->full[st], STAGE);
                    tma_load_3d(d, &tmK, &bars->full[st], 0, it.h, t);
                    tma_load_3d(d + KH_BYTES, &tmK, &bars->full[st], 64, it.h, t);
                    tma_load_3d_hint(d + K_BYTES, &tmV, &bars->full[st], DV * it.half, it.h, t, once);
                    issued = kc + 1;
                }
                it.next(p);
            }
            if (!ok) {
                for (uint32_t i = (issued > NKV ? issued - NKV : 0); i < issued; ++i) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&bars->full[i % NKV], (i / NKV) & 1) && globaltimer_ns() - t0 < 100000000ull) {}
                }
            }
        }
    } else if (warp == 1) {
        // ================================================================ tcgen05 issuer
        if (lane == 0) {
            const uint64_t dkt = sdesc_sw128(smem_u32(smem), KH_BYTES, 1024);
            const uint64_t dv = sdesc_sw128(smem_u32(smem + K_BYTES), V_BYTES, 1024);
            Item it;
            it.init(p);
            bool ok = true;
            uint32_t nfix = 0;                    // partial chunks handed to warp 2 so far
            while (ok && it.valid) {
                if (it.nch > 0) {
                    const uint32_t ab_i = it.a & 1;
                    if (!wait_bar(&bars->acc_empty[ab_i], ((it.a >> 1) & 1) ^ 1, ab)) { ok = false; break; }
                    for (int c = 0; c < it.nch; ++c) {
                        const uint32_t kc = it.kc0 + c, st = kc % NKV;
                        if (!wait_bar(&bars->full[st], (kc / NKV) & 1, ab)) { ok = false; break; }
                        // a partial last chunk: warp 2 zeroes its tail rows first
                        if (c == it.nch - 1 && it.len % KC != 0) {
                            mbar_arrive(&bars->fix_req);
                            if (!wait_bar(&bars->fix_done, nfix & 1, ab)) { ok = false; break; }
                            ++nfix;
                        }
                        tc_fence_after();
                        const uint64_t a = dkt + ((st * STAGE) >> 4), b = dv + ((st * STAGE) >> 4);
#pragma unroll
                        for (int s = 0; s < KC / 16; ++s)
                            mma_ss(tmem + ab_i * DV, a + ((s * 2048) >> 4), b + ((s * 2048) >> 4), IDESC_KV,
                                   (c > 0 || s > 0));
                        tc_commit(&bars->empty[st]);
                    }
                    if (!ok) break;
                    tc_commit(&bars->acc_full[ab_i]);
                }
                it.next(p);
            }
            tc_commit(&bars->drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars->drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {}
        }
    } else if (warp == 2) {
        // ================================================================ tail rows of a partial chunk
        Item it;
        it.init(p);
        bool ok = true;
        uint32_t nfix = 0;
        while (ok && it.valid) {
            const int rem = it.len % KC;
            if (it.nch > 0 && rem != 0) {
                // the issuer asks once the chunk has landed
                const uint32_t kc = it.kc0 + it.nch - 1, st = kc % NKV;
                if (!warp_all(wait_bar(&bars->fix_req, nfix & 1, ab))) { ok = false; break; }
                ++nfix;
                // V rows are 128 contiguous bytes each (row r at r * 128 in the swizzled tile)
                uint4* vrows = reinterpret_cast<uint4*>(smem + st * STAGE + K_BYTES);
                for (int i = rem * 8 + lane; i < KC * 8; i += 32) vrows[i] = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
                mbar_arrive(&bars->fix_done);
            }
            it.next(p);
        }
    } else if (warp >= 4) {
        // ================================================================ accumulator -> state rows
        const int quad = warp & 3;
        const int m = quad * 32 + lane;                  // state row (key index i)
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        Item it;
        it.init(p);
        bool ok = true;
        while (ok && it.valid) {
            float x[DV];
            if (it.nch > 0) {
                const uint32_t ab_i = it.a & 1;
                if (!warp_all(wait_bar(&bars->acc_full[ab_i], (it.a >> 1) & 1, ab))) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t r[32];
                    tmem_ld_x32(tmem + lane_base + ab_i * DV + 32 * hh, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) x[32 * hh + q] = __uint_as_float(r[q]);
                }
                tc_fence_before();
                mbar_arrive(&bars->acc_empty[ab_i]);
            } else {
#pragma unroll
                for (int q = 0; q < DV; ++q) x[q] = 0.f;
            }
            const int64_t row = (((int64_t)it.seq * p.H + it.h) * D + m) * D + DV * it.half;
            if (p.init) {
                const float4* s0 = reinterpret_cast<const float4*>(p.init + row);
#pragma unroll
                for (int q = 0; q < DV / 4; ++q) {
                    const float4 v = __ldg(s0 + q);
                    x[4 * q] += v.x; x[4 * q + 1] += v.y; x[4 * q + 2] += v.z; x[4 * q + 3] += v.w;
                }
            }
            float4* dst = reinterpret_cast<float4*>(p.out + row);
#pragma unroll
            for (int q = 0; q < DV / 4; ++q) dst[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            it.next(p);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace state
}  // namespace la
