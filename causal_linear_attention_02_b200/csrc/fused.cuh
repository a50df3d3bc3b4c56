// Single-pass Lightning Attention prefill for bf16, d = 128, B in {128, 256}.
//
// Method (page "MiniMax-01 Lightning Attention", section "Lightning Attention
// 设计"; page "首个线性注意力架构的大模型来了…", section "4.1 创新的线性注意力"):
//   O_b = (Q_b K_b^T, causal mask) V_b  +  Q_b . KV_prefix(b),
//   KV_prefix(b) = S0 + sum_{c<b} K_c^T V_c.
// The across-block prefix is the "AllGather + local prefix sum" of the page
// "MiniMax-01 Lightning Attention", section "计算优化" (LASP+), done here inside
// one GPU as a single-pass scan with decoupled look-back (Merrill & Garland,
// "Single-pass Parallel Prefix Scan with Decoupled Look-back", 2016): each
// tile publishes its block state U_b = K_b^T V_b as soon as the tensor cores
// have it, and finds its exclusive prefix by walking back over its
// predecessors' published inclusive prefixes or aggregates.
//
// One persistent CTA per SM, tiles t = (block g, head h), g-major, taken
// round-robin (t = blockIdx.x, blockIdx.x + gridDim.x, ...). A tile is B
// query rows processed as R = B/128 sub-units of 128 rows, last sub-unit
// first (it streams every key chunk of the block and so computes U_b on the
// way). Roles (320 threads):
//   warp 0     TMA producer: Q sub-unit tiles and 64-token K/V chunks
//   warp 1     tcgen05 issuer: S = Q K^T, O += P V, U += K^T V, O += Q prefix
//   warps 2-5  scores -> P (mask, bf16, written back into TMEM); publish U_b
//   warps 6-9  look-back -> bf16 prefix in shared memory; store the inclusive
//              prefix; O epilogue (TMEM -> bf16 -> global)
//   warp 10    publisher: one lane per flag kind makes the stored states visible
//              (gpu-scope fence after the group's mbarrier arrive) and raises
//              the flags, so no worker group stalls on a memory fence
//   warp 11    idle (keeps three warps per sub-partition for the register budget)
// Published states live in a small ring of W slots per (sequence, head) so
// they stay resident in L2; a slot is reused only after every tile that may
// read it has finished its look-back (look-back depth is bounded by L = W - 2).
// Every wait is bounded (globaltimer); on expiry the CTA records
// LA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace la {
namespace fused {

using namespace la::sm100;

constexpr int D = 128;
constexpr int UM = 128;                    // rows per sub-unit (MMA M)
constexpr int KC = 64;                     // keys per chunk
constexpr int NQ = 3;                      // Q sub-unit stages
constexpr int NKV = 3;                     // K/V chunk stages
constexpr int W = kStateSlots;             // published-state ring slots per chain
constexpr int L = W - 2;                   // look-back depth: blocks b-1 .. b-L may be read
static_assert(L == 2, "the look-back below reads at most incl(b-1), or agg(b-1) + incl(b-2)");

constexpr uint32_t Q_BYTES = UM * D * 2;   // 32 KB
constexpr uint32_t QH_BYTES = UM * 64 * 2; // 16 KB (one 64-column half)
constexpr uint32_t KV_BYTES = KC * D * 2;  // 16 KB
constexpr uint32_t KVH_BYTES = KC * 64 * 2;
constexpr uint32_t PRE_BYTES = D * D * 2;  // 32 KB
constexpr uint32_t PREH_BYTES = D * 64 * 2;

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_KV = OFF_Q + NQ * Q_BYTES;
constexpr uint32_t OFF_PRE = OFF_KV + NKV * 2 * KV_BYTES;
constexpr uint32_t OFF_BAR = OFF_PRE + PRE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;

constexpr uint32_t TM_O = 0, TM_S = 256, TM_U = 384, TM_COLS = 512;

constexpr uint32_t IDESC_S = idesc_bf16(128, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, false, true);
constexpr uint32_t IDESC_QP = idesc_bf16(128, 128, false, true);
constexpr uint32_t IDESC_KV = idesc_bf16(128, 128, true, true);

constexpr int NTHREADS = 384;

struct Bars {
    uint64_t q_full[NQ], q_empty[NQ];
    uint64_t kv_full[NKV], kv_empty[NKV];
    uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
    uint64_t pre_full, pre_empty, u_full, u_empty, drain;
    uint64_t grp_a, grp_b;     // bounded 128-thread group barriers of warps 2-5 and 6-9
    uint64_t lbd_st, agg_st, incl_st;     // worker group -> publisher: look-back reads done / state stored
    uint64_t lbd_pub, agg_pub, incl_pub;  // publisher -> worker group: flag released
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

struct Params {
    __nv_bfloat16* out;
    const BlockEntry* table;
    const Control* ctrl;
    int* agg_flag;      // [block][H]   1 once the block's aggregate is published
    int* incl_flag;     // [block][H]   1 once its inclusive prefix is published
    int* lb_done;       // [block][H]   1 once its look-back no longer reads anything
    float* states;      // [slot][H][2][D*D] (0: aggregate, 1: inclusive), element (i,j) at ((j/4)*D + i)*4 + j%4
    const float* init;  // [nseq][H][D][D] row-major, or nullptr
    int H;
    int R;              // sub-units per tile (B / 128)
    uint64_t wait_ns;
    long long suppress_tile;   // test hook: this tile publishes nothing (-1: none)
    uint64_t* trace;           // optional [tile][kTraceEvents] globaltimer stamps, or nullptr
};

// Phase stamps of the optional per-tile trace (la_debug_set_trace).
enum TraceEvent {
    TR_MMA_START = 0,     // issuer: tile's first Q stage ready
    TR_MMA_CHUNKS = 1,    // issuer: every chunk MMA of the tile issued
    TR_MMA_PREFIX = 2,    // issuer: prefix available, inter-block MMAs issued
    TR_LB_START = 3,      // look-back group: look-back begins
    TR_LB_END = 4,        // look-back group: exclusive prefix in registers
    TR_PREFIX = 5,        // look-back group: bf16 prefix written to shared memory
    TR_INCL = 6,          // look-back group: inclusive prefix published
    TR_EPI_END = 7,       // look-back group: O stored
    TR_AGG = 8,           // P group: aggregate published
    TR_P_END = 9,         // P group: last P of the tile written
    TR_KV0 = 10,          // issuer: first K/V chunk of the tile ready
    TR_OEMPTY_A = 11,     // issuer: O buffer of the first sub-unit free
    TR_OEMPTY_B = 12,     // issuer: O buffer of the second sub-unit free
    TR_P0 = 13,           // issuer: P of the first chunk ready
    TR_PLAST = 14,        // issuer: P of the first sub-unit's last chunk ready
    TR_LOAD0 = 15,        // producer: first load of the tile issued
    kTraceEvents = 16
};
#define LA_TRACE(t, ev)                                                         \
    do {                                                                       \
        if (p.trace) p.trace[(int64_t)(t) * kTraceEvents + (ev)] = globaltimer_ns(); \
    } while (0)

struct Tile {
    int g, h;
    BlockEntry e;
};

__device__ __forceinline__ Tile tile_of(int64_t t, const Params& p) {
    Tile x;
    x.g = (int)(t / p.H);
    x.h = (int)(t % p.H);
    x.e = p.table[x.g];
    return x;
}
__device__ __forceinline__ int sub_rows(const Tile& x, int r) { return min(UM, x.e.len - UM * r); }
__device__ __forceinline__ int sub_chunks(const Tile& x, int r) {
    return min((r + 1) * (UM / KC), (x.e.len + KC - 1) / KC);
}
__device__ __forceinline__ bool owns_state(const Tile& x) { return !x.e.last; }

__device__ __forceinline__ float* slot_ptr(const Params& p, const Tile& x, int blk, int which) {
    const int64_t slot = (int64_t)x.e.slot0 + (blk % W);
    return p.states + ((slot * p.H + x.h) * 2 + which) * (int64_t)(D * D);
}

// Warp-uniform AND: every decision that guards a .sync.aligned tcgen05
// instruction must be the same in all 32 lanes, even on an abort path.
__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x) != 0; }

__device__ __forceinline__ int ld_acquire(const int* ptr) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}
__device__ __forceinline__ int ld_relaxed(const int* ptr) {
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void st_release(int* ptr, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" :: "l"(ptr), "r"(v) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t c0, int32_t c1, int32_t c2, uint64_t pol) {
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                 " [%0], [%1, {%3, %4, %5}], [%2], %6;"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
                    "r"(c0), "r"(c1), "r"(c2), "l"(pol)
                 : "memory");
}

// Abort state of one launch: a CTA-local flag in shared memory and a
// launch-wide flag in the workspace. The first wait that runs out of time
// raises both (and records LA_ERR_TIMEOUT); every other wait of every CTA
// then gives up at its next check, so the launch ends promptly.
struct Abort {
    volatile int* cta;
    volatile int* global;
    uint64_t limit_ns;
    __device__ __forceinline__ bool raised() const { return *cta || *global; }
    __device__ __forceinline__ void raise() const {
        if (!*cta) { *cta = 1; *global = 1; record_status(LA_ERR_TIMEOUT); }
    }
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Abort& ab) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (ab.raised()) { *ab.cta = 1; return false; }
            if (globaltimer_ns() - t0 > ab.limit_ns) { ab.raise(); return false; }
        }
    }
}

__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int32_t c0, int32_t c1, int32_t c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2) : "memory");
}

// Bounded spin until *flag becomes nonzero. False on timeout or abort.
__device__ __forceinline__ bool spin_flag(const int* flag, const Abort& ab) {
    if (ld_acquire(flag)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ld_acquire(flag)) return true;
        if ((it & 15u) == 0) {
            if (ab.raised()) { *ab.cta = 1; return false; }
            if (globaltimer_ns() - t0 > ab.limit_ns) { ab.raise(); return false; }
            __nanosleep(64);
        }
    }
}

// A slot is rewritten only after every tile that may still read its previous
// occupant (block b - W, read by the look-backs of blocks b-W+1 .. b-W+L) has
// finished its look-back. With W = L + 2 the newest of those is two blocks
// back, so publishing never waits on the look-back of the block just before.
// Called by one thread; the caller shares the outcome through a group barrier.
__device__ __forceinline__ bool wait_reclaim(const Params& p, const Tile& x, const Abort& ab) {
    const int blk = x.e.blk;
    for (int c = max(0, blk - W + 1); c <= blk - W + L; ++c) {
        const int gc = x.g - (blk - c);
        if (!spin_flag(p.lb_done + (int64_t)gc * p.H + x.h, ab)) return false;
    }
    return true;
}
// Early, non-blocking probe of the same condition (relaxed loads issued at the
// start of a tile, consumed much later). A true result still needs an acquire
// fence before the slot is written; a false result falls back to wait_reclaim.
__device__ __forceinline__ bool probe_reclaim(const Params& p, const Tile& x) {
    const int blk = x.e.blk;
    int all = 1;
    for (int c = max(0, blk - W + 1); c <= blk - W + L; ++c)
        all &= ld_relaxed(p.lb_done + (int64_t)(x.g - (blk - c)) * p.H + x.h);
    return all != 0;
}

// Bounded barrier of one 128-thread group built on an mbarrier (arrive, then
// wait for the phase). Unlike bar.sync it cannot hang if a member has left
// after an abort: the wait gives up at the time limit. Returns false then.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, const Abort& ab) {
    mbar_arrive(bar);
    const bool ok = wait_bar(bar, phase, ab);
    phase ^= 1u;
    return ok;
}

__global__ void __launch_bounds__(NTHREADS, 1)
prefill_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&bars->abort_flag, const_cast<volatile int*>(&p.ctrl->abort), p.wait_ns};

    if (threadIdx.x == 0) {
        for (int i = 0; i < NQ; ++i) { mbar_init(&bars->q_full[i], 1); mbar_init(&bars->q_empty[i], 1); }
        for (int i = 0; i < NKV; ++i) { mbar_init(&bars->kv_full[i], 1); mbar_init(&bars->kv_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);  mbar_init(&bars->p_full[i], 128);
            mbar_init(&bars->o_full[i], 1);  mbar_init(&bars->o_empty[i], 128);
        }
        mbar_init(&bars->pre_full, 128);
        mbar_init(&bars->pre_empty, 1);
        mbar_init(&bars->u_full, 1);
        mbar_init(&bars->u_empty, 256);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->grp_a, 128);
        mbar_init(&bars->grp_b, 128);
        mbar_init(&bars->lbd_st, 128);
        mbar_init(&bars->agg_st, 128);
        mbar_init(&bars->incl_st, 128);
        mbar_init(&bars->lbd_pub, 1);
        mbar_init(&bars->agg_pub, 1);
        mbar_init(&bars->incl_pub, 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQ); prefetch_tmap(&tmK); prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const int64_t ntiles = p.ctrl->ok ? (int64_t)p.ctrl->nblocks * p.H : 0;
    const int R = p.R;

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            uint32_t q_it = 0, kv_it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                const Tile x = tile_of(t, p);
                // stage the next tile of this CTA in L2 a whole tile ahead, so that the
                // shared-memory loads below (and the next tile's) hit L2
                if (t + gridDim.x < ntiles) {
                    const Tile y = tile_of(t + gridDim.x, p);
                    for (int r = R - 1; r >= 0; --r) {
                        if (sub_rows(y, r) <= 0) continue;
                        tma_prefetch_l2_3d(&tmQ, 0, y.h, y.e.tok0 + UM * r);
                        tma_prefetch_l2_3d(&tmQ, 64, y.h, y.e.tok0 + UM * r);
                    }
                    int rf = R - 1;                       // first sub-unit streamed (most chunks)
                    while (rf > 0 && sub_rows(y, rf) <= 0) --rf;
                    const int nk = sub_chunks(y, rf);
                    for (int j = 0; j < nk; ++j) {
                        const int tk = y.e.tok0 + KC * j;
                        tma_prefetch_l2_3d(&tmK, 0, y.h, tk);
                        tma_prefetch_l2_3d(&tmK, 64, y.h, tk);
                        tma_prefetch_l2_3d(&tmV, 0, y.h, tk);
                        tma_prefetch_l2_3d(&tmV, 64, y.h, tk);
                    }
                }
                for (int r = R - 1; ok && r >= 0; --r) {
                    if (sub_rows(x, r) <= 0) continue;
                    const uint32_t qs = q_it % NQ;
                    if (!wait_bar(&bars->q_empty[qs], ((q_it / NQ) & 1) ^ 1, ab)) { ok = false; break; }
                    uint8_t* qd = smem + OFF_Q + qs * Q_BYTES;
                    const int tq = x.e.tok0 + UM * r;
                    if (r == R - 1 || sub_rows(x, R - 1) <= 0) LA_TRACE(t, TR_LOAD0);
                    mbar_expect_tx(&bars->q_full[qs], Q_BYTES);
                    tma_load_3d_hint(qd, &tmQ, &bars->q_full[qs], 0, x.h, tq, pol);
                    tma_load_3d_hint(qd + QH_BYTES, &tmQ, &bars->q_full[qs], 64, x.h, tq, pol);
                    ++q_it;
                    const int nkc = sub_chunks(x, r);
                    for (int j = 0; j < nkc; ++j) {
                        const uint32_t st = kv_it % NKV;
                        if (!wait_bar(&bars->kv_empty[st], ((kv_it / NKV) & 1) ^ 1, ab)) { ok = false; break; }
                        uint8_t* kd = smem + OFF_KV + st * 2 * KV_BYTES;
                        uint8_t* vd = kd + KV_BYTES;
                        const int tk = x.e.tok0 + KC * j;
                        // chunks re-streamed by a later sub-unit of the same block stay in L2
                        const uint64_t pk = (r == R - 1 && R > 1 && j < (R - 1) * (UM / KC)) ? 0 : pol;
                        mbar_expect_tx(&bars->kv_full[st], 2 * KV_BYTES);
                        if (pk) {
                            tma_load_3d_hint(kd, &tmK, &bars->kv_full[st], 0, x.h, tk, pk);
                            tma_load_3d_hint(kd + KVH_BYTES, &tmK, &bars->kv_full[st], 64, x.h, tk, pk);
                            tma_load_3d_hint(vd, &tmV, &bars->kv_full[st], 0, x.h, tk, pk);
                            tma_load_3d_hint(vd + KVH_BYTES, &tmV, &bars->kv_full[st], 64, x.h, tk, pk);
                        } else {
                            tma_load_3d(kd, &tmK, &bars->kv_full[st], 0, x.h, tk);
                            tma_load_3d(kd + KVH_BYTES, &tmK, &bars->kv_full[st], 64, x.h, tk);
                            tma_load_3d(vd, &tmV, &bars->kv_full[st], 0, x.h, tk);
                            tma_load_3d(vd + KVH_BYTES, &tmV, &bars->kv_full[st], 64, x.h, tk);
                        }
                        ++kv_it;
                    }
                }
            }
            // On abort, wait (bounded) for the copies still in flight into this CTA's
            // shared memory: only the latest load of each stage can be pending.
            if (!ok) {
                for (uint32_t i = (q_it > NQ ? q_it - NQ : 0); i < q_it; ++i) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&bars->q_full[i % NQ], (i / NQ) & 1) &&
                           globaltimer_ns() - t0 < 100000000ull) {}
                }
                for (uint32_t i = (kv_it > NKV ? kv_it - NKV : 0); i < kv_it; ++i) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&bars->kv_full[i % NKV], (i / NKV) & 1) &&
                           globaltimer_ns() - t0 < 100000000ull) {}
                }
            }
        }
    } else if (warp == 1) {
        // ================================================================ tcgen05 issuer
        if (lane == 0) {
            uint32_t q_it = 0, kv_it = 0, s_it = 0, o_it = 0, u_it = 0, tile_it = 0;
            const uint32_t q_base = smem_u32(smem + OFF_Q);
            const uint32_t kv_base = smem_u32(smem + OFF_KV);
            const uint32_t pre_base = smem_u32(smem + OFF_PRE);
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                const Tile x = tile_of(t, p);
                const bool own = owns_state(x);
                uint32_t sub_q[2], sub_o[2];
                int nsub = 0;
                for (int r = R - 1; ok && r >= 0; --r) {
                    if (sub_rows(x, r) <= 0) continue;
                    const int nkc = sub_chunks(x, r);
                    const bool with_u = own && r == R - 1;
                    const uint32_t qs = q_it % NQ, ob = o_it & 1;
                    if (!wait_bar(&bars->q_full[qs], (q_it / NQ) & 1, ab)) { ok = false; break; }
                    if (nsub == 0) LA_TRACE(t, TR_MMA_START);
                    tc_fence_after();
                    const uint32_t qa = q_base + qs * Q_BYTES;
                    const uint32_t d_o = tmem + TM_O + ob * 128;
                    auto issue_scores = [&](int j) -> bool {
                        const uint32_t kvi = kv_it + j, st = kvi % NKV;
                        if (!wait_bar(&bars->kv_full[st], (kvi / NKV) & 1, ab)) return false;
                        if (nsub == 0 && j == 0) LA_TRACE(t, TR_KV0);
                        tc_fence_after();
                        const uint32_t kb = kv_base + st * 2 * KV_BYTES;
                        const uint32_t d_s = tmem + TM_S + ((s_it + j) & 1) * 64;
#pragma unroll
                        for (int s = 0; s < D / 16; ++s)
                            mma_ss(d_s, sdesc_sw128(qa + (s >> 2) * QH_BYTES + (s & 3) * 32, 16, 1024),
                                   sdesc_sw128(kb + (s >> 2) * KVH_BYTES + (s & 3) * 32, 16, 1024), IDESC_S, s > 0);
                        tc_commit(&bars->s_full[(s_it + j) & 1]);
                        return true;
                    };
                    if (!issue_scores(0)) { ok = false; break; }
                    if (!wait_bar(&bars->o_empty[ob], ((o_it >> 1) & 1) ^ 1, ab)) { ok = false; break; }
                    LA_TRACE(t, nsub == 0 ? TR_OEMPTY_A : TR_OEMPTY_B);
                    if (with_u && !wait_bar(&bars->u_empty, (u_it & 1) ^ 1, ab)) { ok = false; break; }
                    tc_fence_after();
                    for (int j = 0; j < nkc; ++j) {
                        if (j + 1 < nkc && !issue_scores(j + 1)) { ok = false; break; }
                        const uint32_t sb = (s_it + j) & 1;
                        if (!wait_bar(&bars->p_full[sb], ((s_it + j) >> 1) & 1, ab)) { ok = false; break; }
                        if (nsub == 0 && j == 0) LA_TRACE(t, TR_P0);
                        if (nsub == 0 && j + 1 == nkc) LA_TRACE(t, TR_PLAST);
                        tc_fence_after();
                        const uint32_t st = (kv_it + j) % NKV;
                        const uint32_t kb = kv_base + st * 2 * KV_BYTES, vb = kb + KV_BYTES;
                        const uint32_t a_p = tmem + TM_S + sb * 64;
#pragma unroll
                        for (int s = 0; s < KC / 16; ++s)
                            mma_ts(d_o, a_p + s * 8, sdesc_sw128(vb + s * 2048, KVH_BYTES, 1024), IDESC_PV,
                                   (j > 0 || s > 0));
                        if (with_u) {
#pragma unroll
                            for (int s = 0; s < KC / 16; ++s)
                                mma_ss(tmem + TM_U, sdesc_sw128(kb + s * 2048, KVH_BYTES, 1024),
                                       sdesc_sw128(vb + s * 2048, KVH_BYTES, 1024), IDESC_KV, (j > 0 || s > 0));
                        }
                        tc_commit(&bars->kv_empty[st]);
                    }
                    if (!ok) break;
                    if (with_u) { tc_commit(&bars->u_full); ++u_it; }
                    kv_it += nkc;
                    s_it += nkc;
                    sub_q[nsub] = qs;
                    sub_o[nsub] = ob;
                    ++nsub;
                    ++q_it;
                    ++o_it;
                }
                if (!ok) break;
                // inter-block right product once the look-back has produced the prefix
                LA_TRACE(t, TR_MMA_CHUNKS);
                if (!wait_bar(&bars->pre_full, tile_it & 1, ab)) { ok = false; break; }
                LA_TRACE(t, TR_MMA_PREFIX);
                tc_fence_after();
                for (int n = 0; n < nsub; ++n) {
                    const uint32_t qa = q_base + sub_q[n] * Q_BYTES;
                    const uint32_t d_o = tmem + TM_O + sub_o[n] * 128;
#pragma unroll
                    for (int s = 0; s < D / 16; ++s)
                        mma_ss(d_o, sdesc_sw128(qa + (s >> 2) * QH_BYTES + (s & 3) * 32, 16, 1024),
                               sdesc_sw128(pre_base + s * 2048, PREH_BYTES, 1024), IDESC_QP, 1);
                    tc_commit(&bars->q_empty[sub_q[n]]);
                    tc_commit(&bars->o_full[sub_o[n]]);
                }
                tc_commit(&bars->pre_empty);
                ++tile_it;
            }
            // every MMA issued by this thread has completed once `drain` fires
            tc_commit(&bars->drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars->drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {}
        }
    } else if (warp < 6) {
        // ================================================================ scores -> P; publish U_b
        const int quad = warp & 3;
        const int m = quad * 32 + lane;
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        const int wt = threadIdx.x - 64;                  // 0..127 within this group
        uint32_t s_it = 0, u_it = 0, grp_phase = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
            const Tile x = tile_of(t, p);
            const bool own = owns_state(x);
            const bool slot_free = (own && wt == 0) ? probe_reclaim(p, x) : true;
            for (int r = R - 1; ok && r >= 0; --r) {
                if (sub_rows(x, r) <= 0) continue;
                const int nkc = sub_chunks(x, r);
                const int qi = UM * r + m;                // query position in the block
                for (int j = 0; j < nkc; ++j, ++s_it) {
                    const uint32_t sb = s_it & 1;
                    if (!warp_all(wait_bar(&bars->s_full[sb], (s_it >> 1) & 1, ab))) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t ts = tmem + lane_base + TM_S + sb * 64;
                    uint32_t a[32], b[32], pk[32];
                    tmem_ld_x32(ts, a);
                    tmem_ld_x32(ts + 32, b);
                    tmem_wait_ld();
                    const int lim = qi - KC * j;          // key column c is kept when c <= lim
                    if (lim >= KC - 1) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            pk[c] = pack_bf16x2(__uint_as_float(a[2 * c]), __uint_as_float(a[2 * c + 1]));
                            pk[16 + c] = pack_bf16x2(__uint_as_float(b[2 * c]), __uint_as_float(b[2 * c + 1]));
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            pk[c] = pack_bf16x2(2 * c <= lim ? __uint_as_float(a[2 * c]) : 0.f,
                                                2 * c + 1 <= lim ? __uint_as_float(a[2 * c + 1]) : 0.f);
                            pk[16 + c] = pack_bf16x2(32 + 2 * c <= lim ? __uint_as_float(b[2 * c]) : 0.f,
                                                     33 + 2 * c <= lim ? __uint_as_float(b[2 * c + 1]) : 0.f);
                        }
                    }
                    tmem_st_x32(ts, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&bars->p_full[sb]);
                    if (wt == 0 && r == 0 && j + 1 == nkc) LA_TRACE(t, TR_P_END);
                }
                if (!ok) break;
                if (own && r == R - 1) {
                    // store the aggregate U_b = K_b^T V_b of this (block, head); the
                    // publisher lane raises its flag once the stores are visible
                    if (!wait_bar(&bars->u_full, u_it & 1, ab)) ok = false;
                    tc_fence_after();
                    if (ok && wt == 0) {
                        if (slot_free) fence_acq_rel_gpu();
                        else if (!wait_reclaim(p, x, ab)) ok = false;
                    }
                    if (!group_sync(&bars->grp_a, grp_phase, ab) || ab.raised()) ok = false;
                    if (ok && !wait_bar(&bars->agg_pub, (u_it & 1) ^ 1, ab)) ok = false;
                    ok = warp_all(ok);
                    if (ok && t != p.suppress_tile) {
                        float* dst = slot_ptr(p, x, x.e.blk, 0);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            uint32_t u[16];
                            tmem_ld_x16(tmem + lane_base + TM_U + 16 * c, u);
                            tmem_wait_ld();
#pragma unroll
                            for (int w = 0; w < 4; ++w)
                                __stcg(reinterpret_cast<float4*>(dst + ((4 * c + w) * D + m) * 4),
                                       make_float4(__uint_as_float(u[4 * w]), __uint_as_float(u[4 * w + 1]),
                                                   __uint_as_float(u[4 * w + 2]), __uint_as_float(u[4 * w + 3])));
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&bars->u_empty);
                    mbar_arrive(&bars->agg_st);
                    ++u_it;
                }
            }
        }
    } else if (warp < 10) {
        // ================================================================ look-back, prefix, inclusive, epilogue
        const int quad = warp & 3;
        const int m = quad * 32 + lane;                   // state row / O row owned by this thread
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        const int wt = threadIdx.x - 192;
        uint32_t tile_it = 0, o_it = 0, u_it = 0, grp_phase = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
            const Tile x = tile_of(t, p);
            const bool own = owns_state(x);
            float4 acc[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            // ---- decoupled look-back: excl(b) = S0 + sum_{c<b} U_c
            if (wt == 0) LA_TRACE(t, TR_LB_START);
            const bool slot_free = (own && wt == 0) ? probe_reclaim(p, x) : true;
            {
                // Depth L = 2: either incl(b-1), or agg(b-1) + incl(b-2); near the
                // sequence start agg(b-1) (+ S0). Lane 0 of each warp polls the
                // flags with relaxed loads issued together, decides, and every lane
                // then takes an acquire fence before reading the chosen states.
                const int blk = x.e.blk;
                int srcs = 0;               // bit 0: incl(b-1), bit 1: agg(b-1), bit 2: incl(b-2), bit 3: S0
                if (blk == 0) {
                    srcs = 8;
                } else if (lane == 0) {
                    const int64_t f1 = (int64_t)(x.g - 1) * p.H + x.h;
                    const int64_t f2 = (int64_t)(x.g - 2) * p.H + x.h;
                    const uint64_t t0 = globaltimer_ns();
                    for (uint32_t it = 0;; ++it) {
                        const int i1 = ld_relaxed(p.incl_flag + f1);
                        const int a1 = ld_relaxed(p.agg_flag + f1);
                        const int i2 = blk >= 2 ? ld_relaxed(p.incl_flag + f2) : 0;
                        if (i1) { srcs = 1; break; }
                        if (a1 && blk == 1) { srcs = 2 | 8; break; }
                        if (a1 && i2) { srcs = 2 | 4; break; }
                        if ((it & 7u) == 7u) {
                            if (ab.raised()) { *ab.cta = 1; srcs = -1; break; }
                            if (globaltimer_ns() - t0 > ab.limit_ns) { ab.raise(); srcs = -1; break; }
                            __nanosleep(32);
                        }
                    }
                    // acquire: the flags seen above synchronise with their release stores;
                    // __syncwarp then orders this before every lane's reads of the states
                    fence_acq_rel_gpu();
                }
                __syncwarp();
                srcs = __shfl_sync(0xffffffffu, srcs, 0);
                if (srcs < 0) ok = false;
                if (ok) {
                    if (srcs & 1) {
                        const float* src = slot_ptr(p, x, blk - 1, 1);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (k * D + m) * 4));
                            acc[k].x += v.x; acc[k].y += v.y; acc[k].z += v.z; acc[k].w += v.w;
                        }
                    }
                    if (srcs & 2) {
                        const float* src = slot_ptr(p, x, blk - 1, 0);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (k * D + m) * 4));
                            acc[k].x += v.x; acc[k].y += v.y; acc[k].z += v.z; acc[k].w += v.w;
                        }
                    }
                    if (srcs & 4) {
                        const float* src = slot_ptr(p, x, blk - 2, 1);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const float4 v = __ldcg(reinterpret_cast<const float4*>(src + (k * D + m) * 4));
                            acc[k].x += v.x; acc[k].y += v.y; acc[k].z += v.z; acc[k].w += v.w;
                        }
                    }
                    if ((srcs & 8) && p.init) {
                        const float4* s0 = reinterpret_cast<const float4*>(
                            p.init + (((int64_t)x.e.seq * p.H + x.h) * D + m) * D);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const float4 v = __ldg(s0 + k);
                            acc[k].x += v.x; acc[k].y += v.y; acc[k].z += v.z; acc[k].w += v.w;
                        }
                    }
                }
                // every read of the predecessors' states is done: let the publisher say so
                if (ok && !wait_bar(&bars->lbd_pub, (tile_it & 1) ^ 1, ab)) ok = false;
                ok = warp_all(ok);
                if (ok) mbar_arrive(&bars->lbd_st);
            }
            if (!ok) break;
            // ---- bf16 prefix into shared memory (MN-major, 128-byte swizzle: row m = key index i)
            if (!warp_all(wait_bar(&bars->pre_empty, (tile_it & 1) ^ 1, ab))) { ok = false; break; }
            {
                uint8_t* pre = smem + OFF_PRE;
#pragma unroll
                for (int jg = 0; jg < 16; ++jg) {
                    const float4 lo = acc[2 * jg], hi = acc[2 * jg + 1];
                    uint4 w;
                    w.x = pack_bf16x2(lo.x, lo.y); w.y = pack_bf16x2(lo.z, lo.w);
                    w.z = pack_bf16x2(hi.x, hi.y); w.w = pack_bf16x2(hi.z, hi.w);
                    const uint32_t off = (jg >> 3) * PREH_BYTES + (m >> 3) * 1024 + (m & 7) * 128 +
                                         (((jg & 7) ^ (m & 7)) << 4);
                    *reinterpret_cast<uint4*>(pre + off) = w;
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars->pre_full);
                if (wt == 0) LA_TRACE(t, TR_PREFIX);
            }
            // ---- inclusive prefix incl(b) = excl(b) + U_b (the publisher raises its flag)
            if (own) {
                if (!wait_bar(&bars->u_full, u_it & 1, ab)) ok = false;
                tc_fence_after();
                if (ok && wt == 0) {
                    if (slot_free) fence_acq_rel_gpu();
                    else if (!wait_reclaim(p, x, ab)) ok = false;
                }
                if (!group_sync(&bars->grp_b, grp_phase, ab) || ab.raised()) ok = false;
                if (ok && !wait_bar(&bars->incl_pub, (u_it & 1) ^ 1, ab)) ok = false;
                ok = warp_all(ok);
                if (ok && t != p.suppress_tile) {
                    float* dst = slot_ptr(p, x, x.e.blk, 1);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t u[16];
                        tmem_ld_x16(tmem + lane_base + TM_U + 16 * c, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const float4 a = acc[4 * c + w];
                            __stcg(reinterpret_cast<float4*>(dst + ((4 * c + w) * D + m) * 4),
                                   make_float4(a.x + __uint_as_float(u[4 * w]), a.y + __uint_as_float(u[4 * w + 1]),
                                               a.z + __uint_as_float(u[4 * w + 2]), a.w + __uint_as_float(u[4 * w + 3])));
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->u_empty);
                if (ok) mbar_arrive(&bars->incl_st);
                ++u_it;
                if (!ok) break;
            }
            // ---- O epilogue of each sub-unit, in the order the MMA warp finishes them
            for (int r = R - 1; ok && r >= 0; --r) {
                const int rows = sub_rows(x, r);
                if (rows <= 0) continue;
                const uint32_t ob = o_it & 1;
                if (!warp_all(wait_bar(&bars->o_full[ob], (o_it >> 1) & 1, ab))) { ok = false; break; }
                tc_fence_after();
                const bool valid = m < rows;
                __nv_bfloat16* orow = p.out + ((int64_t)(x.e.tok0 + UM * r + m) * p.H + x.h) * D;
                // drain the whole accumulator row (packed to bf16 on the way) and free
                // the TMEM buffer at once, so the next sub-unit's P.V can start while
                // these rows are stored
                uint32_t pk[64];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t v0[32];
                    tmem_ld_x32(tmem + lane_base + TM_O + ob * 128 + 32 * c4, v0);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        pk[16 * c4 + c] = pack_bf16x2(__uint_as_float(v0[2 * c]), __uint_as_float(v0[2 * c + 1]));
                }
                tc_fence_before();
                mbar_arrive(&bars->o_empty[ob]);
                ++o_it;
                if (valid) {
#pragma unroll
                    for (int w = 0; w < 16; ++w)
                        __stcs(reinterpret_cast<uint4*>(orow + 8 * w),
                               make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]));
                }
            }
            if (wt == 0) LA_TRACE(t, TR_EPI_END);
            ++tile_it;
        }
    } else if (warp == 10 && lane == 0) {
        // ================================================================ publisher
        // Three in-order streams (look-back done, aggregate stored, inclusive stored),
        // polled round robin without blocking. For each completed item: the worker
        // group's mbarrier arrive released its stores at CTA scope; the release
        // store below makes them visible at gpu scope together with the flag.
        int64_t t_lb = blockIdx.x, t_ag = blockIdx.x, t_in = blockIdx.x;
        uint32_t n_lb = 0, n_ag = 0, n_in = 0;
        auto next_own = [&](int64_t t) {
            while (t < ntiles && !owns_state(tile_of(t, p))) t += gridDim.x;
            return t;
        };
        t_ag = next_own(t_ag);
        t_in = next_own(t_in);
        uint64_t t0 = globaltimer_ns();
        while (t_lb < ntiles || t_ag < ntiles || t_in < ntiles) {
            bool any = false;
            if (t_lb < ntiles && mbar_try_wait(&bars->lbd_st, n_lb & 1)) {
                const Tile x = tile_of(t_lb, p);
                st_release(p.lb_done + (int64_t)x.g * p.H + x.h, 1);
                LA_TRACE(t_lb, TR_LB_END);
                mbar_arrive(&bars->lbd_pub);
                ++n_lb; t_lb += gridDim.x; any = true;
            }
            if (t_ag < ntiles && mbar_try_wait(&bars->agg_st, n_ag & 1)) {
                const Tile x = tile_of(t_ag, p);
                if (t_ag != p.suppress_tile) {
                    st_release(p.agg_flag + (int64_t)x.g * p.H + x.h, 1);
                    LA_TRACE(t_ag, TR_AGG);
                }
                mbar_arrive(&bars->agg_pub);
                ++n_ag; t_ag = next_own(t_ag + gridDim.x); any = true;
            }
            if (t_in < ntiles && mbar_try_wait(&bars->incl_st, n_in & 1)) {
                const Tile x = tile_of(t_in, p);
                if (t_in != p.suppress_tile) {
                    st_release(p.incl_flag + (int64_t)x.g * p.H + x.h, 1);
                    LA_TRACE(t_in, TR_INCL);
                }
                mbar_arrive(&bars->incl_pub);
                ++n_in; t_in = next_own(t_in + gridDim.x); any = true;
            }
            if (any) {
                t0 = globaltimer_ns();
            } else {
                if (ab.raised()) break;
                if (globaltimer_ns() - t0 > ab.limit_ns) { ab.raise(); break; }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace fused
}  // namespace la
