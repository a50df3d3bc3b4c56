// Block table and block-state prefix scan.
//
// The method cuts every sequence into blocks of B tokens (page "首个线性注意力
// 架构的大模型来了…", section "4.1 创新的线性注意力": 序列划分) and carries a
// compact d x d prefix state from block to block (双阶段计算, 区块间处理). Packed
// varlen sequences are independent ("data packing", page "MiniMax-01 Lightning
// Attention", section "计算优化"), so blocks restart at every sequence start.
#pragma once

#include "common.cuh"
#include "decay.cuh"

namespace la {

// Block-wide exclusive scan over a 1024-thread CTA; returns the exclusive
// prefix of `x` and adds the CTA total to `carry` (shared, read by all).
__device__ __forceinline__ int32_t cta_exclusive_scan(int32_t x, int32_t* warp_sums, int32_t* carry) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int32_t incl = x;
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int32_t w = lane < nw ? warp_sums[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_sums[lane] = w;
    }
    __syncthreads();
    const int32_t excl = *carry + (wid > 0 ? warp_sums[wid - 1] : 0) + incl - x;
    __syncthreads();
    if (threadIdx.x == 0) *carry += warp_sums[nw - 1];
    __syncthreads();
    return excl;
}

// Validates cu_seqlens and writes, per sequence s,
//   seq_blk[s]  = sum_{s' < s} ceil(len_s' / B)            (first global block)
//   seq_slot[s] = sum_{s' < s} min(nblocks_s' - 1, W)      (first published-state slot)
// and the totals at index nseq. One CTA of 1024 threads. cu == nullptr means
// one sequence of T tokens.
__global__ void __launch_bounds__(1024) seq_blocks_kernel(const int32_t* __restrict__ cu, int nseq,
                                                          int64_t T, int B, int32_t* __restrict__ seq_blk,
                                                          int32_t* __restrict__ seq_slot,
                                                          Control* __restrict__ ctrl) {
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry_b, carry_s;
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0) { carry_b = 0; carry_s = 0; bad = 0; }
    __syncthreads();
    // validation: cu[0] = 0, non-decreasing, cu[nseq] = T
    if (cu != nullptr) {
        for (int s = tid; s < nseq; s += blockDim.x)
            if (cu[s + 1] < cu[s]) bad = 1;
        if (tid == 0 && (cu[0] != 0 || (int64_t)cu[nseq] != T)) bad = 1;
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            ctrl->nblocks = 0;
            ctrl->ok = 0;
            ctrl->nslots = 0;
            ctrl->abort = 0;
            record_status(LA_ERR_BAD_SEQLENS);
        }
        return;
    }
    for (int base = 0; base < nseq; base += blockDim.x) {
        const int s = base + tid;
        int32_t nb = 0;
        if (s < nseq) {
            const int64_t len = cu ? (int64_t)(cu[s + 1] - cu[s]) : T;
            nb = (int32_t)((len + B - 1) / B);
        }
        const int32_t ns = nb > 1 ? min(nb - 1, kStateSlots) : 0;
        const int32_t eb = cta_exclusive_scan(nb, warp_sums, &carry_b);
        const int32_t es = cta_exclusive_scan(ns, warp_sums, &carry_s);
        if (s < nseq) {
            seq_blk[s] = eb;
            seq_slot[s] = es;
        }
    }
    if (tid == 0) {
        seq_blk[nseq] = carry_b;
        seq_slot[nseq] = carry_s;
        ctrl->nblocks = carry_b;
        ctrl->ok = 1;
        ctrl->nslots = carry_s;
        ctrl->abort = 0;
        ctrl->ticket = 0;       // the single-pass prefill's tile tickets
    }
}

// One thread per possible block: finds its sequence by binary search over
// seq_blk, writes the BlockEntry and clears the block's `nflags` per-head
// flag words (flags: [nflag_arrays][max_blocks][H] int32, may be null).
__global__ void fill_block_table_kernel(const int32_t* __restrict__ cu, int nseq, int64_t T, int B,
                                        const int32_t* __restrict__ seq_blk,
                                        const int32_t* __restrict__ seq_slot,
                                        const Control* __restrict__ ctrl,
                                        BlockEntry* __restrict__ table, int64_t max_blocks,
                                        int32_t* __restrict__ flags, int nflag_arrays, int H) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= max_blocks || g >= ctrl->nblocks) return;
    int lo = 0, hi = nseq - 1;          // last s with seq_blk[s] <= g
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seq_blk[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int32_t b = (int32_t)(g - seq_blk[s]);
    const int64_t start = cu ? (int64_t)cu[s] : 0;
    const int64_t len = cu ? (int64_t)(cu[s + 1] - cu[s]) : T;
    BlockEntry e;
    e.seq = s;
    e.blk = b;
    e.tok0 = (int32_t)(start + (int64_t)b * B);
    const int64_t rest = len - (int64_t)b * B;
    e.len = (int32_t)(rest < B ? rest : B);
    e.last = (g + 1 == seq_blk[s + 1]) ? 1 : 0;
    e.slot0 = seq_slot ? seq_slot[s] : 0;
    e.pad[0] = e.pad[1] = 0;
    table[g] = e;
    for (int a = 0; a < nflag_arrays; ++a)
        for (int h = 0; h < H; ++h) flags[((int64_t)a * max_blocks + g) * H + h] = 0;
}

// Sequences longest first, so that work items of equal cost start together
// and the longest chains start first. Sorted by counting when nseq is at
// most kSortMax (ties keep their input order), else left in input order.
constexpr int kSortMax = 2048;

// Validates cu_seqlens like seq_blocks_kernel and writes, per sequence,
// its first token and length (seqs) and the processing order (order,
// longest first). One CTA of 1024 threads. cu == nullptr means one
// sequence of T tokens.
__global__ void __launch_bounds__(1024) seq_table_kernel(const int32_t* __restrict__ cu, int nseq, int64_t T,
                                                         SeqEntry* __restrict__ seqs,
                                                         int32_t* __restrict__ order,
                                                         Control* __restrict__ ctrl) {
    __shared__ int32_t lens[kSortMax];
    __shared__ int bad, nmulti, nsingle;
    const int tid = threadIdx.x;
    if (tid == 0) { bad = 0; nmulti = 0; nsingle = 0; }
    __syncthreads();
    if (cu != nullptr) {
        for (int s = tid; s < nseq; s += blockDim.x)
            if (cu[s + 1] < cu[s]) bad = 1;
        if (tid == 0 && (cu[0] != 0 || (int64_t)cu[nseq] != T)) bad = 1;
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            ctrl->nblocks = 0;
            ctrl->ok = 0;
            ctrl->nslots = 0;
            ctrl->abort = 0;
            record_status(LA_ERR_BAD_SEQLENS);
        }
        return;
    }
    const bool sort = nseq <= kSortMax;
    for (int s = tid; s < nseq; s += blockDim.x) {
        SeqEntry e;
        e.tok0 = cu ? cu[s] : 0;
        e.len = cu ? cu[s + 1] - cu[s] : (int32_t)T;
        seqs[s] = e;
        if (sort) lens[s] = e.len;
        else order[s] = s;
        if (e.len >= 2) atomicAdd(&nmulti, 1);
        else if (e.len == 1) atomicAdd(&nsingle, 1);
    }
    __syncthreads();
    if (sort) {
        for (int s = tid; s < nseq; s += blockDim.x) {
            const int32_t l = lens[s];
            int rank = 0;
            for (int t = 0; t < nseq; ++t) {
                const int32_t lt = lens[t];
                rank += (lt > l) || (lt == l && t < s);
            }
            order[rank] = s;
        }
    }
    if (tid == 0) {
        ctrl->nblocks = 0;
        ctrl->ok = 1;
        ctrl->nslots = 0;
        ctrl->abort = 0;
        // longest first puts the sequences of two or more tokens first and the one-token
        // sequences right after them; unsorted, every sequence stays in the first group
        ctrl->nmulti = sort ? nmulti : nseq;
        ctrl->nsingle = sort ? nsingle : 0;
        ctrl->ticket = 0;
    }
}

// Exclusive prefix over the blocks of every (sequence, head) chain:
//   prefix[g] = S0 + sum_{blocks c of the same sequence before g} U[c]
// and, optionally, the chain total S0 + sum_all U into state_out. With a
// per-head decay rate (decay != nullptr; decay.cuh) the running state is
// multiplied by lambda^len(g) before U[g] is added.
// U, prefix: [block][H][d*d]; init, state_out: [nseq][H][d*d].
// grid = (ceil(d*d / 1024), nseq * H), 256 threads, 4 consecutive elements per thread.
template <typename OutT>
__global__ void __launch_bounds__(256) chain_scan_kernel(const float* __restrict__ U,
                                                         OutT* __restrict__ prefix,
                                                         const float* init, float* state_out,
                                                         const int32_t* __restrict__ seq_blk,
                                                         const Control* __restrict__ ctrl,
                                                         int nseq, int H, int dd, bool skip_last,
                                                         const BlockEntry* __restrict__ table, const float* decay) {
    if (!ctrl->ok) return;
    const int chain = blockIdx.y;
    const int s = chain / H, h = chain % H;
    float l2 = 0.f;
    if (decay && !load_decay(decay, h, l2)) return;
    const int e = (blockIdx.x * 256 + threadIdx.x) * 4;
    if (e >= dd) return;
    const int64_t g0 = seq_blk[s], g1 = seq_blk[s + 1];
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    if (init) run = *reinterpret_cast<const float4*>(init + ((int64_t)s * H + h) * dd + e);
    const int64_t gend = skip_last ? g1 - 1 : g1;   // the last block's U is not needed by a prefill
    float4 nxt = make_float4(0.f, 0.f, 0.f, 0.f);
    if (g0 < gend) nxt = __ldcs(reinterpret_cast<const float4*>(U + ((int64_t)g0 * H + h) * dd + e));
    for (int64_t g = g0; g < g1; ++g) {
        if (prefix) {
            OutT* p = prefix + ((int64_t)g * H + h) * dd + e;
            if constexpr (sizeof(OutT) == 4) {
                *reinterpret_cast<float4*>(p) = run;
            } else {
                uint2 w;
                w.x = pack_bf16x2(run.x, run.y);
                w.y = pack_bf16x2(run.z, run.w);
                *reinterpret_cast<uint2*>(p) = w;
            }
        }
        if (g < gend) {
            const float4 u = nxt;
            if (g + 1 < gend)
                nxt = __ldcs(reinterpret_cast<const float4*>(U + ((int64_t)(g + 1) * H + h) * dd + e));
            if (decay) {
                const float w = decay_pow(l2, table[g].len);
                run.x = fmaf(w, run.x, u.x); run.y = fmaf(w, run.y, u.y);
                run.z = fmaf(w, run.z, u.z); run.w = fmaf(w, run.w, u.w);
            } else {
                run.x += u.x; run.y += u.y; run.z += u.z; run.w += u.w;
            }
        }
    }
    if (state_out) *reinterpret_cast<float4*>(state_out + ((int64_t)s * H + h) * dd + e) = run;
}

// Final states of the empty sequences for la_prefill_with_state (the prefill
// kernel visits only sequences with tokens): S0, or zero without one. A CTA
// takes one sequence at a time and copies its [H][d][d] state in 16-byte
// groups; sequences with tokens cost one length read. Nothing when the call's
// checks failed (ctrl->ok = 0).
__global__ void __launch_bounds__(256)
empty_states_kernel(const SeqEntry* seqs, int nseq, int64_t per_seq4, const float4* init, float4* out,
                    const Control* ctrl) {
    if (!ctrl->ok) return;
    // a CTA per empty sequence at a time; sequences with tokens are skipped whole
    for (int s = blockIdx.x; s < nseq; s += gridDim.x) {
        if (seqs[s].len > 0) continue;
        const int64_t base = (int64_t)s * per_seq4;
        for (int64_t i = threadIdx.x; i < per_seq4; i += blockDim.x)
            out[base + i] = init ? init[base + i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

}  // namespace la
