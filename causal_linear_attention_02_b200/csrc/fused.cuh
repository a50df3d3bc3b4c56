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
// One persistent CTA per SM, tiles t = (block g, head h), g-major, taken by
// atomic ticket in that order (see kTileRing). A tile is B
// query rows processed as R = B/128 sub-units of 128 rows, last sub-unit
// first (it streams every key chunk of the block and so computes U_b on the
// way). Roles (512 threads, 128 registers each):
//   warp 0       TMA producer: Q sub-unit tiles and 64-token K/V chunks
//   warp 1       tcgen05 issuer: U += K^T V, S = Q K^T, O += P V, O += Q prefix
//   warp 2       publisher: makes stored states visible at gpu scope and raises
//                their flags; grants ring slots (no worker group waits on a fence)
//   warp 3       spare
//   warps 4-7    scores -> P (mask, bf16, written back into TMEM); store U_b
//   warps 8-11   columns 0..63 and warps 12-15 columns 64..127 of: look-back ->
//                bf16 prefix in shared memory; inclusive prefix = exclusive +
//                U_b (read back from the stored aggregate); O epilogue (TMA store)
// Published states live in a small ring of W slots per (sequence, head) so
// they stay resident in L2; a slot is reused only after every tile that may
// read it has finished its look-back (look-back depth is bounded by L = W - 2).
// Every wait is bounded (globaltimer); on expiry the CTA records
// LA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "sm100.cuh"
#include "pipe.cuh"

namespace la {
namespace fused {

using namespace la::sm100;

constexpr int D = 128;
constexpr int UM = 128;                    // rows per sub-unit (MMA M)
constexpr int KC = 64;                     // keys per chunk
#ifndef LA_FUSED_NQ
#define LA_FUSED_NQ 3
#endif
#ifndef LA_FUSED_NKV
#define LA_FUSED_NKV 3
#endif
#ifndef LA_FUSED_KV_PREFETCH
#define LA_FUSED_KV_PREFETCH 1
#endif
constexpr int NQ = LA_FUSED_NQ;            // Q sub-unit stages
constexpr int NKV = LA_FUSED_NKV;          // K/V chunk stages
static_assert(NQ * 32 + NKV * 32 + 32 <= 224, "shared memory: Q stages + K/V stages + prefix buffer");
constexpr int W = kStateSlots;             // published-state ring slots per chain
constexpr int L = 3;                       // look-back depth: blocks b-1 .. b-L may be read
static_assert(W >= L + 2, "slot reuse must not wait on the look-back of the block just before");

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
constexpr uint32_t SMEM_BYTES = OFF_BAR + 1024 + 1024;   // barriers and tile ring + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

constexpr uint32_t TM_O = 0, TM_S = 256, TM_U = 384, TM_COLS = 512;

constexpr uint32_t IDESC_S = idesc_bf16(128, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, false, true);
constexpr uint32_t IDESC_QP = idesc_bf16(128, 128, false, true);
constexpr uint32_t IDESC_KV = idesc_bf16(128, 128, true, true);

constexpr int NTHREADS = 512;
// Tiles are taken by atomic ticket in tile order (block-major, head fastest), so every
// predecessor of a tile (same head, earlier block: a smaller ticket) belongs to a CTA that
// was already running when this one drew it. Forward progress then never depends on CTAs
// that are not resident (another stream's kernel may hold SMs). The producer draws each
// tile when it first needs it, at most two ahead of the one it loads, and hands the
// sequence to the other roles through a small ring; roles lag the producer by a few
// tiles at most, far less than the ring holds.
constexpr uint32_t kTileRing = 32;

struct Bars {
    uint64_t q_full[NQ], q_empty[NQ];
    uint64_t kv_full[NKV], kv_empty[NKV];
    uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
    uint64_t pre_full, pre_empty, u_full, u_empty, drain;
    uint64_t grp_a;            // bounded 128-thread barrier of the P / epilogue group
    uint64_t stage_done;       // P group -> column groups: O stores have read the staging buffer
    uint64_t lbd_st, incl_st;             // worker group -> publisher: look-back reads done / incl stored
    uint64_t agg_st[2];                   // P group -> publisher and column groups: aggregate stored
                                          // (two, used alternately: the P group runs one tile ahead)
    uint64_t lbd_pub;                     // publisher -> look-back group: previous look-back flag released
    uint64_t incl_pub;                    // publisher -> column groups: previous inclusive flag released
    uint64_t slot_ok;                     // publisher -> P group: this tile's ring slot may be written
    uint32_t tmem_base;
    int abort_flag;
    int32_t tile_ring[kTileRing];         // the CTA's k-th tile at [k % kTileRing], drawn by the producer
    int32_t tile_tag[kTileRing];          // k of the entry (a stale entry is an error, never used)
    uint32_t drawn;                       // tiles drawn so far
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

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
    uint64_t grace_ns;         // look-back: how long to wait for incl(b-1) before reading agg(b-1) + incl(b-2)
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
    TR_B_INCL_ST = 16,    // column group 0: inclusive prefix stored, handed to the publisher
    TR_B_LBD_ST = 17,     // column group 0: look-back reads done, handed to the publisher
    TR_A_AGG_ST = 18,     // P group: aggregate stored, handed to the publisher
    TR_PUB_INCL = 19,     // publisher: inclusive hand-off seen (before its release store)
    TR_B_LB_DECIDED = 20, // column group 0: look-back sources decided
    TR_A_EPI1_FULL = 21,  // P group: first epilogue sub-unit accumulator complete
    TR_A_EPI1_FREE = 22,  // P group: first epilogue sub-unit accumulator released
    TR_A_U_FULL = 23,     // P group: next tile's block state complete in TMEM
    TR_A_SLOT_OK = 24,    // P group: next tile's ring slot granted
    TR_A_EPI0_FULL = 25,  // P group: second epilogue sub-unit accumulator complete
    TR_A_EPI0_FREE = 26,  // P group: second epilogue sub-unit accumulator released
    TR_A_S0 = 27,         // P group: scores of the tile's first chunk seen
    TR_PUB_AGG = 28,      // publisher: aggregate hand-off seen (before its release store)
    TR_A_SJ = 32,         // + j (j < 4): P group, scores of chunk j of the first sub-unit seen
    TR_A_PJ = 36,         // + j: P group, P of chunk j of the first sub-unit written
    TR_I_SJ = 40,         // + j: issuer, score MMAs of chunk j of the first sub-unit issued
    TR_I_PVJ = 44,        // + j: issuer, PV MMAs of chunk j of the first sub-unit issued
    kTraceEvents = 48
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
// fp32 state rows: L2-only (.cg) 16-byte accesses with an L2 eviction-priority hint.
__device__ __forceinline__ float4 ld_state4(const float* ptr, uint64_t pol) {
    float4 v;
    asm volatile("ld.global.cg.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(ptr), "l"(pol) : "memory");
    return v;
}
__device__ __forceinline__ void st_state4(float* ptr, float4 v, uint64_t pol) {
    asm volatile("st.global.cg.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;"
                 :: "l"(ptr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol) : "memory");
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

// The CTA's k-th tile from the ring (ntiles when the tickets have run out). Blocking
// (bounded) until the producer has drawn it; a ring entry of another k means a role fell
// further behind than the ring holds: the launch gives up (LA_ERR_TIMEOUT) rather than
// use it.
__device__ __noinline__ bool ring_tile(Bars* bars, uint32_t k, int64_t ntiles, const Abort ab, int64_t& t) {
    const volatile uint32_t* drawn = &bars->drawn;
    if (*drawn <= k) {
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 1; *drawn <= k; ++it) {
            if ((it & 31u) == 0) {
                if (ab.raised()) { *ab.cta = 1; return false; }
                if (globaltimer_ns() - t0 > ab.limit_ns) { ab.raise(); return false; }
            }
        }
    }
    const volatile int32_t* ring = bars->tile_ring;
    const volatile int32_t* tag = bars->tile_tag;
    const int32_t v = ring[k % kTileRing];
    if ((uint32_t)tag[k % kTileRing] != k) { ab.raise(); return false; }
    t = v < ntiles ? (int64_t)v : ntiles;
    return true;
}
// Non-blocking: -1 while the producer has not drawn tile k yet.
__device__ __forceinline__ int64_t ring_peek(Bars* bars, uint32_t k, int64_t ntiles) {
    if (*reinterpret_cast<const volatile uint32_t*>(&bars->drawn) <= k) return -1;
    const int32_t v = reinterpret_cast<const volatile int32_t*>(bars->tile_ring)[k % kTileRing];
    return v < ntiles ? (int64_t)v : ntiles;
}

// Ring-slot reuse: block b writes slot b % W, last used by block b - W, which
// the look-backs of blocks b-W+1 .. b-W+L may read. With W = L + 2 the newest
// of those is two blocks back, so the check (made by the publisher lane) never
// waits on the look-back of the block just before.

__global__ void __launch_bounds__(NTHREADS, 1)
prefill_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const Params p) {
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
        mbar_init(&bars->pre_full, 256);
        mbar_init(&bars->pre_empty, 1);
        mbar_init(&bars->u_full, 1);
        mbar_init(&bars->u_empty, 128);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->grp_a, 128);
        mbar_init(&bars->stage_done, 1);
        mbar_init(&bars->lbd_st, 256);
        mbar_init(&bars->agg_st[0], 128);
        mbar_init(&bars->agg_st[1], 128);
        mbar_init(&bars->incl_st, 256);
        mbar_init(&bars->lbd_pub, 1);
        mbar_init(&bars->incl_pub, 1);
        mbar_init(&bars->slot_ok, 1);
        bars->abort_flag = 0;
        bars->drawn = 0;
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
        // Per tile: first the whole K and V of this CTA's NEXT tile (its block state
        // U is computed one tile ahead, see the issuer), then Q and the K/V chunks
        // of this tile's sub-units. The lookahead load brings the next tile's K/V
        // into L2, where its own pass finds it a tile later.
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();    // last read of a Q / K / V tile
            const uint64_t keep = policy_evict_last();    // K / V tiles that are read again soon
            uint32_t q_it = 0, kv_it = 0;
            bool ok = true;
            auto load_chunk = [&](const Tile& y, int j, uint64_t hint) -> bool {
                const uint32_t st = kv_it % NKV;
                if (!wait_bar(&bars->kv_empty[st], ((kv_it / NKV) & 1) ^ 1, ab)) return false;
                uint8_t* kd = smem + OFF_KV + st * 2 * KV_BYTES;
                uint8_t* vd = kd + KV_BYTES;
                const int tk = y.e.tok0 + KC * j;
                mbar_expect_tx(&bars->kv_full[st], 2 * KV_BYTES);
                if (hint) {
                    tma_load_3d_hint(kd, &tmK, &bars->kv_full[st], 0, y.h, tk, hint);
                    tma_load_3d_hint(kd + KVH_BYTES, &tmK, &bars->kv_full[st], 64, y.h, tk, hint);
                    tma_load_3d_hint(vd, &tmV, &bars->kv_full[st], 0, y.h, tk, hint);
                    tma_load_3d_hint(vd + KVH_BYTES, &tmV, &bars->kv_full[st], 64, y.h, tk, hint);
                } else {
                    tma_load_3d(kd, &tmK, &bars->kv_full[st], 0, y.h, tk);
                    tma_load_3d(kd + KVH_BYTES, &tmK, &bars->kv_full[st], 64, y.h, tk);
                    tma_load_3d(vd, &tmV, &bars->kv_full[st], 0, y.h, tk);
                    tma_load_3d(vd + KVH_BYTES, &tmV, &bars->kv_full[st], 64, y.h, tk);
                }
                ++kv_it;
                return true;
            };
            auto load_lookahead = [&](int64_t tt) -> bool {
                if (tt >= ntiles) return true;
                const Tile y = tile_of(tt, p);
                if (!owns_state(y)) return true;
                for (int j = 0; j < R * (UM / KC); ++j)
                    if (!load_chunk(y, j, keep)) return false;   // read again by the tile itself
                return true;
            };
            // draws the CTA's tiles 0..k (tile tickets, see kTileRing) and returns tile k
            Control* ctrl_w = const_cast<Control*>(p.ctrl);
            volatile uint32_t* drawn = &bars->drawn;
            volatile int32_t* ring = bars->tile_ring;
            volatile int32_t* tag = bars->tile_tag;
            auto tile_k = [&](uint32_t k) -> int64_t {
                while (*drawn <= k) {
                    const uint32_t n = *drawn;
                    const int v = atomicAdd(&ctrl_w->ticket, 1);
                    ring[n % kTileRing] = v;
                    tag[n % kTileRing] = (int32_t)n;
                    __threadfence_block();
                    *drawn = n + 1;
                }
                const int32_t v = ring[k % kTileRing];
                return v < ntiles ? (int64_t)v : ntiles;
            };
            if (!load_lookahead(tile_k(0))) ok = false;
            for (uint32_t k = 0; ok; ++k) {
                const int64_t t = tile_k(k);
                if (t >= ntiles) break;
                const Tile x = tile_of(t, p);
                const int64_t t1 = tile_k(k + 1);
                if (t1 < ntiles) {                     // the next tile's Q into L2 a tile ahead
                    const Tile y = tile_of(t1, p);
                    for (int r = R - 1; r >= 0; --r) {
                        if (sub_rows(y, r) <= 0) continue;
                        tma_prefetch_l2_3d(&tmQ, 0, y.h, y.e.tok0 + UM * r);
                        tma_prefetch_l2_3d(&tmQ, 64, y.h, y.e.tok0 + UM * r);
                    }
                }
                const int64_t t2 = LA_FUSED_KV_PREFETCH ? tile_k(k + 2) : ntiles;
                if (t2 < ntiles) {
                    // K / V of the tile after next into L2, ahead of its look-ahead loads
                    const Tile y = tile_of(t2, p);
                    if (owns_state(y)) {
                        for (int j = 0; j < R * (UM / KC); ++j) {
                            const int tk = y.e.tok0 + KC * j;
                            tma_prefetch_l2_3d(&tmK, 0, y.h, tk);
                            tma_prefetch_l2_3d(&tmK, 64, y.h, tk);
                            tma_prefetch_l2_3d(&tmV, 0, y.h, tk);
                            tma_prefetch_l2_3d(&tmV, 64, y.h, tk);
                        }
                    }
                }
                if (!load_lookahead(t1)) { ok = false; break; }
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
                        // chunks re-streamed by a later sub-unit of the same block stay in L2
                        const bool again = r == R - 1 && R > 1 && j < (R - 1) * (UM / KC);
                        if (!load_chunk(x, j, again ? keep : pol)) { ok = false; break; }
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
            // Block state of tile tt, one tile ahead: U = sum over its chunks of K^T V,
            // accumulated in TMEM as the chunks land; u_full fires when it is complete.
            auto lookahead_state = [&](int64_t tt) -> bool {
                if (tt >= ntiles) return true;
                const Tile y = tile_of(tt, p);
                if (!owns_state(y)) return true;
                if (!wait_bar(&bars->u_empty, (u_it & 1) ^ 1, ab)) return false;  // previous U drained
                for (int j = 0; j < R * (UM / KC); ++j, ++kv_it) {
                    const uint32_t st = kv_it % NKV;
                    if (!wait_bar(&bars->kv_full[st], (kv_it / NKV) & 1, ab)) return false;
                    tc_fence_after();
                    const uint32_t kb = kv_base + st * 2 * KV_BYTES, vb = kb + KV_BYTES;
#pragma unroll
                    for (int s = 0; s < KC / 16; ++s)
                        mma_ss(tmem + TM_U, sdesc_sw128(kb + s * 2048, KVH_BYTES, 1024),
                               sdesc_sw128(vb + s * 2048, KVH_BYTES, 1024), IDESC_KV, (j > 0 || s > 0));
                    tc_commit(&bars->kv_empty[st]);
                }
                tc_commit(&bars->u_full);
                ++u_it;
                return true;
            };
            int64_t tnext = ntiles;
            if (!ring_tile(bars, 0, ntiles, ab, tnext) || !lookahead_state(tnext)) ok = false;
            for (uint32_t k = 0; ok && tnext < ntiles; ++k) {
                const int64_t t = tnext;
                const Tile x = tile_of(t, p);
                if (!ring_tile(bars, k + 1, ntiles, ab, tnext) || !lookahead_state(tnext)) { ok = false; break; }
                uint32_t sub_q[2], sub_o[2];
                int nsub = 0;
                for (int r = R - 1; ok && r >= 0; --r) {
                    if (sub_rows(x, r) <= 0) continue;
                    const int nkc = sub_chunks(x, r);
                    const uint32_t qs = q_it % NQ, ob = o_it & 1;
                    if (!wait_bar(&bars->q_full[qs], (q_it / NQ) & 1, ab)) { ok = false; break; }
                    if (nsub == 0) LA_TRACE(t, TR_MMA_START);
                    tc_fence_after();
                    const uint32_t qa = q_base + qs * Q_BYTES;
                    const uint32_t d_o = tmem + TM_O + ob * 128;
                    auto issue_scores = [&](int j) -> bool {
                        const uint32_t kvi = kv_it + j, st = kvi % NKV;
                        if (!wait_bar(&bars->kv_full[st], (kvi / NKV) & 1, ab)) return false;
                        tc_fence_after();
                        const uint32_t kb = kv_base + st * 2 * KV_BYTES;
                        const uint32_t d_s = tmem + TM_S + ((s_it + j) & 1) * 64;
#pragma unroll
                        for (int s = 0; s < D / 16; ++s)
                            mma_ss(d_s, sdesc_sw128(qa + (s >> 2) * QH_BYTES + (s & 3) * 32, 16, 1024),
                                   sdesc_sw128(kb + (s >> 2) * KVH_BYTES + (s & 3) * 32, 16, 1024), IDESC_S, s > 0);
                        tc_commit(&bars->s_full[(s_it + j) & 1]);
                        if (nsub == 0 && j < 4) LA_TRACE(t, TR_I_SJ + j);
                        return true;
                    };
                    if (!issue_scores(0)) { ok = false; break; }
                    if (!wait_bar(&bars->o_empty[ob], ((o_it >> 1) & 1) ^ 1, ab)) { ok = false; break; }
                    LA_TRACE(t, nsub == 0 ? TR_OEMPTY_A : TR_OEMPTY_B);
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
                        tc_commit(&bars->kv_empty[st]);
                        if (nsub == 0 && j < 4) LA_TRACE(t, TR_I_PVJ + j);
                    }
                    if (!ok) break;
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
    } else if (warp >= 4 && warp < 8) {
        // ================================================================ scores -> P; store U of the next tile
        const int quad = warp & 3;
        const int m = quad * 32 + lane;
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        const int wt = threadIdx.x - 128;                 // 0..127 within this group
        uint32_t s_it = 0, u_it = 0, o_it = 0, tile_it = 0, grp_phase = 0;
        bool ok = true;
        const uint64_t keep = policy_evict_last();       // published states stay in L2
        const uint64_t o_pol = policy_evict_first();     // O is never read back
        // Store the block state of tile tt (computed one tile ahead by the issuer) as
        // the aggregate of its ring slot; the publisher raises its flag.
        auto store_aggregate = [&](int64_t tt) -> bool {
            if (tt >= ntiles) return true;
            const Tile y = tile_of(tt, p);
            if (!owns_state(y)) return true;
            if (!warp_all(wait_bar(&bars->u_full, u_it & 1, ab))) return false;
            if (wt == 0) LA_TRACE(tt, TR_A_U_FULL);
            tc_fence_after();
            if (!warp_all(wait_bar(&bars->slot_ok, u_it & 1, ab))) return false;   // ring slot is free
            if (wt == 0) LA_TRACE(tt, TR_A_SLOT_OK);
            if (tt != p.suppress_tile) {
                float* dst = slot_ptr(p, y, y.e.blk, 0);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t u[16];
                    tmem_ld_x16(tmem + lane_base + TM_U + 16 * c, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        st_state4(dst + ((4 * c + w) * D + m) * 4,
                                  make_float4(__uint_as_float(u[4 * w]), __uint_as_float(u[4 * w + 1]),
                                              __uint_as_float(u[4 * w + 2]), __uint_as_float(u[4 * w + 3])),
                                  keep);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->u_empty);
            mbar_arrive(&bars->agg_st[u_it & 1]);
            if (wt == 0) LA_TRACE(tt, TR_A_AGG_ST);
            ++u_it;
            return true;
        };
        int64_t tnext = ntiles;
        ok = warp_all(ring_tile(bars, 0, ntiles, ab, tnext));
        if (ok && !store_aggregate(tnext)) ok = false;
        for (uint32_t k = 0; ok && tnext < ntiles; ++k) {
            const int64_t t = tnext;
            const Tile x = tile_of(t, p);
            if (!warp_all(ring_tile(bars, k + 1, ntiles, ab, tnext))) { ok = false; break; }
            for (int r = R - 1; ok && r >= 0; --r) {
                if (sub_rows(x, r) <= 0) continue;
                const int nkc = sub_chunks(x, r);
                const int qi = UM * r + m;                // query position in the block
                for (int j = 0; j < nkc; ++j, ++s_it) {
                    const uint32_t sb = s_it & 1;
                    if (!warp_all(wait_bar(&bars->s_full[sb], (s_it >> 1) & 1, ab))) { ok = false; break; }
                    if (wt == 0 && r == R - 1 && j == 0) LA_TRACE(t, TR_A_S0);
                    if (wt == 0 && r == R - 1 && j < 4) LA_TRACE(t, TR_A_SJ + j);
                    tc_fence_after();
                    const uint32_t ts = tmem + lane_base + TM_S + sb * 64;
                    const int lim = qi - KC * j;          // key column c is kept when c <= lim
                    uint32_t pk[32];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {      // two 32-column halves keep registers low
                        uint32_t a[32];
                        tmem_ld_x32(ts + 32 * hh, a);
                        tmem_wait_ld();
                        if (lim >= KC - 1) {
#pragma unroll
                            for (int c = 0; c < 16; ++c)
                                pk[16 * hh + c] = pack_bf16x2(__uint_as_float(a[2 * c]), __uint_as_float(a[2 * c + 1]));
                        } else {
#pragma unroll
                            for (int c = 0; c < 16; ++c) {
                                const int c0 = 32 * hh + 2 * c;
                                pk[16 * hh + c] = pack_bf16x2(c0 <= lim ? __uint_as_float(a[2 * c]) : 0.f,
                                                              c0 + 1 <= lim ? __uint_as_float(a[2 * c + 1]) : 0.f);
                            }
                        }
                    }
                    tmem_st_x32(ts, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&bars->p_full[sb]);
                    if (wt == 0 && r == 0 && j + 1 == nkc) LA_TRACE(t, TR_P_END);
                    if (wt == 0 && r == R - 1 && j < 4) LA_TRACE(t, TR_A_PJ + j);
                }
            }
            // ---- O epilogue of each sub-unit, in the order the issuer finishes them:
            // drain the accumulator row (packed to bf16) and free it at once; full
            // 128-row sub-units go out as TMA tensor stores staged in the prefix buffer
            // (free once this tile's inter-block MMAs are done), a ragged last sub-unit
            // of a sequence with masked direct stores. The next tile's block state is
            // stored right after the first sub-unit, so the issuer can compute the one
            // after it while the rest of this epilogue runs.
            bool staged = false;
            for (int r = R - 1; ok && r >= 0; --r) {
                const int rows = sub_rows(x, r);
                if (rows <= 0) continue;
                const uint32_t ob = o_it & 1;
                if (!warp_all(wait_bar(&bars->o_full[ob], (o_it >> 1) & 1, ab))) { ok = false; break; }
                if (wt == 0) LA_TRACE(t, r == R - 1 ? TR_A_EPI1_FULL : TR_A_EPI0_FULL);
                tc_fence_after();
                const bool full = rows == UM;
                uint8_t* stage = smem + OFF_PRE;
                if (full) {
                    if (!staged) {            // all inter-block MMAs of this tile have read the prefix
                        if (!warp_all(wait_bar(&bars->pre_empty, tile_it & 1, ab))) { ok = false; break; }
                        staged = true;
                    }
                    if (wt == 0) bulk_wait_read0();              // the previous O store has read the buffer
                    if (!warp_all(group_sync(&bars->grp_a, grp_phase, ab))) { ok = false; break; }
                }
                __nv_bfloat16* orow = p.out + ((int64_t)(x.e.tok0 + UM * r + m) * p.H + x.h) * D;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {      // 32 columns at a time
                    uint32_t v0[32];
                    tmem_ld_x32(tmem + lane_base + TM_O + ob * 128 + 32 * c4, v0);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        pk[c] = pack_bf16x2(__uint_as_float(v0[2 * c]), __uint_as_float(v0[2 * c + 1]));
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int g = 4 * c4 + w;     // 16-byte group of the row
                        const uint4 val = make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
                        if (full)
                            *reinterpret_cast<uint4*>(stage + (g >> 3) * PREH_BYTES + (m >> 3) * 1024 +
                                                      (m & 7) * 128 + (((g & 7) ^ (m & 7)) << 4)) = val;
                        else if (m < rows)
                            __stcs(reinterpret_cast<uint4*>(orow + 8 * g), val);
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->o_empty[ob]);               // the accumulator is free again
                if (wt == 0) LA_TRACE(t, r == R - 1 ? TR_A_EPI1_FREE : TR_A_EPI0_FREE);
                ++o_it;
                if (full) {
                    fence_proxy_async_smem();
                    if (!warp_all(group_sync(&bars->grp_a, grp_phase, ab))) { ok = false; break; }
                    if (wt == 0) {
                        const int tq = x.e.tok0 + UM * r;
                        tma_store_3d_hint(&tmO, stage, 0, x.h, tq, o_pol);
                        tma_store_3d_hint(&tmO, stage + PREH_BYTES, 64, x.h, tq, o_pol);
                        bulk_commit();
                    }
                }
                if (r == R - 1 && ok && !store_aggregate(tnext)) ok = false;
            }
            if (!ok) break;
            if (sub_rows(x, R - 1) <= 0 && !store_aggregate(tnext)) { ok = false; break; }
            // the staging buffer is free for the next prefix once these stores have read it
            if (wt == 0) {
                bulk_wait_read0();
                mbar_arrive(&bars->stage_done);
            }
            if (wt == 0) LA_TRACE(t, TR_EPI_END);
            ++tile_it;
        }
        if (wt == 0) bulk_wait0();            // every O store has landed before the CTA exits
    } else if (warp >= 8) {
        // ================================================================ look-back, prefix, inclusive
        // Two groups, each owning 64 of the 128 state / output columns.
        const int hb = warp >= 12 ? 1 : 0;
        const int kb = 16 * hb;                           // first float4 column group of this half
        const int quad = warp & 3;
        const int m = quad * 32 + lane;                   // state row owned by this thread
        const int wt = threadIdx.x - (hb ? 384 : 256);
        uint8_t* half_buf = smem + OFF_PRE + hb * PREH_BYTES;   // prefix half (O staging between tiles)
        uint32_t tile_it = 0, u_it = 0;
        bool ok = true;
        const uint64_t keep = policy_evict_last();       // published states stay in L2
        auto add_row = [&](float4 (&acc)[16], const float* src) {
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8) {          // 8 loads in flight at a time
                float4 v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    v[k] = ld_state4(src + ((kb + k0 + k) * D + m) * 4, keep);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    acc[k0 + k].x += v[k].x; acc[k0 + k].y += v[k].y;
                    acc[k0 + k].z += v[k].z; acc[k0 + k].w += v[k].w;
                }
            }
        };
        for (uint32_t k = 0; ok; ++k) {
            int64_t t = ntiles;
            if (!warp_all(ring_tile(bars, k, ntiles, ab, t))) { ok = false; break; }
            if (t >= ntiles) break;
            const Tile x = tile_of(t, p);
            const bool own = owns_state(x);
            float4 acc[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            // ---- decoupled look-back: excl(b) = S0 + sum_{c<b} U_c (this group's columns)
            if (wt == 0 && hb == 0) LA_TRACE(t, TR_LB_START);
            {
                // Depth up to L: incl(b-1), or agg(b-1) + incl(b-2), or agg(b-1) + agg(b-2)
                // + incl(b-3), ...; near the sequence start the aggregates down to block 0
                // plus S0. Lane 0 of each warp polls the flags with relaxed loads, prefers
                // incl(b-1) during a grace period, decides, takes an acquire fence;
                // __syncwarp orders it before every lane's reads.
                const int blk = x.e.blk;
                int srcs = 0;               // bits 0-2: aggregates b-1, b-2, ... to add; bit 3: base is S0
                if (blk == 0) {
                    srcs = 8;
                } else if (lane == 0) {
                    const int64_t fb = (int64_t)x.g * p.H + x.h;      // flag index of block b
                    const uint64_t t0 = globaltimer_ns();
                    for (uint32_t it = 0;; ++it) {
                        if (ld_relaxed(p.incl_flag + fb - p.H)) { srcs = 0; break; }
                        if (globaltimer_ns() - t0 > p.grace_ns) {
                            int na = 0;
                            srcs = -2;
                            while (na < L - 1 && na < blk && ld_relaxed(p.agg_flag + fb - (int64_t)(na + 1) * p.H)) {
                                ++na;        // aggregates of blocks b-1 .. b-na are published
                                if (na == blk) { srcs = na | 8; break; }
                                if (ld_relaxed(p.incl_flag + fb - (int64_t)(na + 1) * p.H)) { srcs = na; break; }
                            }
                            if (srcs >= 0) break;
                            srcs = 0;
                        }
                        if ((it & 7u) == 7u) {
                            if (ab.raised()) { *ab.cta = 1; srcs = -1; break; }
                            if (globaltimer_ns() - t0 > ab.limit_ns) { ab.raise(); srcs = -1; break; }
                            __nanosleep(32);
                        }
                    }
                    fence_acq_rel_gpu();
                }
                __syncwarp();
                srcs = __shfl_sync(0xffffffffu, srcs, 0);
                if (wt == 0 && hb == 0) LA_TRACE(t, TR_B_LB_DECIDED);
                if (srcs < 0) ok = false;
                if (ok) {
                    const int na = srcs & 7;
                    for (int c = 1; c <= na; ++c) add_row(acc, slot_ptr(p, x, blk - c, 0));
                    if (!(srcs & 8)) {
                        add_row(acc, slot_ptr(p, x, blk - na - 1, 1));
                    } else if (p.init) {
                        const float4* s0 = reinterpret_cast<const float4*>(
                            p.init + (((int64_t)x.e.seq * p.H + x.h) * D + m) * D) + kb;
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const float4 v = __ldg(s0 + k);
                            acc[k].x += v.x; acc[k].y += v.y; acc[k].z += v.z; acc[k].w += v.w;
                        }
                    }
                }
                // every read of the predecessors' states is done: let the publisher say so
                if (ok && !wait_bar(&bars->lbd_pub, (tile_it & 1) ^ 1, ab)) ok = false;
                ok = warp_all(ok);
                if (ok) mbar_arrive(&bars->lbd_st);
                if (wt == 0 && hb == 0) LA_TRACE(t, TR_B_LBD_ST);
            }
            if (!ok) break;
            // ---- inclusive prefix incl(b) = excl(b) + U_b first (it is on the chain of the
            // next block), with U_b read back from the aggregate the P group stored
            if (own) {
                // aggregate stored (CTA scope); the P group waited for the ring slot before
                // storing it, which also frees the slot's inclusive half
                if (!wait_bar(&bars->agg_st[u_it & 1], (u_it >> 1) & 1, ab)) ok = false;
                ok = warp_all(ok);
                if (ok && t != p.suppress_tile) {          // acc keeps excl(b) for the prefix
                    const float* src = slot_ptr(p, x, x.e.blk, 0);
                    float* dst = slot_ptr(p, x, x.e.blk, 1);
#pragma unroll
                    for (int k0 = 0; k0 < 16; k0 += 8) {
                        float4 v[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            v[k] = ld_state4(src + ((kb + k0 + k) * D + m) * 4, keep);
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float4 a4 = acc[k0 + k];
                            st_state4(dst + ((kb + k0 + k) * D + m) * 4,
                                      make_float4(a4.x + v[k].x, a4.y + v[k].y, a4.z + v[k].z, a4.w + v[k].w),
                                      keep);
                        }
                    }
                }
                // the publisher has taken the previous inclusive prefix (one in flight)
                if (ok && !wait_bar(&bars->incl_pub, (u_it & 1) ^ 1, ab)) ok = false;
                ok = warp_all(ok);
                if (ok) mbar_arrive(&bars->incl_st);
                if (wt == 0 && hb == 0) LA_TRACE(t, TR_B_INCL_ST);
                ++u_it;
                if (!ok) break;
            }
            // ---- bf16 prefix (this group's 64 columns) into its half of the shared
            // buffer (MN-major, 128-byte swizzle, row m = key index i). The buffer also
            // stages O for the previous tile's TMA stores: wait until they have read it.
            if (!warp_all(wait_bar(&bars->pre_empty, (tile_it & 1) ^ 1, ab))) { ok = false; break; }
            if (!warp_all(wait_bar(&bars->stage_done, (tile_it & 1) ^ 1, ab))) { ok = false; break; }
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const float4 lo = acc[2 * g], hi = acc[2 * g + 1];
                uint4 w;
                w.x = pack_bf16x2(lo.x, lo.y); w.y = pack_bf16x2(lo.z, lo.w);
                w.z = pack_bf16x2(hi.x, hi.y); w.w = pack_bf16x2(hi.z, hi.w);
                *reinterpret_cast<uint4*>(half_buf + (m >> 3) * 1024 + (m & 7) * 128 + ((g ^ (m & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->pre_full);
            if (wt == 0 && hb == 0) LA_TRACE(t, TR_PREFIX);
            ++tile_it;
        }
    } else if (warp == 2 && lane == 0) {
        // ================================================================ publisher
        // Four in-order streams polled round robin without blocking:
        //   slot: own tile n may write its ring slot once the tiles that may still
        //         read the slot's previous occupant have finished their look-backs
        //         (acquire loads of their flags); released to the P group through
        //         slot_ok, at most one own tile ahead of it (the column groups write
        //         the slot's inclusive half only after that group's aggregate);
        //   lb / agg / incl: for each completed item the worker group's mbarrier
        //         arrive released its accesses at CTA scope; the release store below
        //         makes them visible at gpu scope together with the flag.
        // Each stream is an index into the CTA's tile sequence; -1: not drawn yet (asked again).
        uint32_t k_lb = 0, k_ag = 0, k_in = 0, k_sl = 0;
        int64_t t_lb = -1, t_ag = -1, t_in = -1, t_sl = -1;
        uint32_t n_lb = 0, n_ag = 0, n_in = 0, n_sl = 0;
        auto own_at = [&](uint32_t& k) -> int64_t {    // the first tile at index >= k with a state of its own
            for (;;) {
                const int64_t t = ring_peek(bars, k, ntiles);
                if (t < 0 || t >= ntiles || owns_state(tile_of(t, p))) return t;
                ++k;
            }
        };
        uint64_t t0 = globaltimer_ns();
        for (;;) {
            if (t_lb < 0) t_lb = ring_peek(bars, k_lb, ntiles);
            if (t_ag < 0) t_ag = own_at(k_ag);
            if (t_in < 0) t_in = own_at(k_in);
            if (t_sl < 0) t_sl = own_at(k_sl);
            if (t_lb >= ntiles && t_ag >= ntiles && t_in >= ntiles) break;
            bool any = false;
            if (t_sl >= 0 && t_sl < ntiles && n_sl <= n_ag) {
                const Tile x = tile_of(t_sl, p);
                const int blk = x.e.blk;
                int free = 1;
                for (int c = max(0, blk - W + 1); c <= blk - W + L; ++c)
                    free &= ld_acquire(p.lb_done + (int64_t)(x.g - (blk - c)) * p.H + x.h);
                if (free) {
                    mbar_arrive(&bars->slot_ok);
                    ++n_sl; ++k_sl; t_sl = -1; any = true;
                }
            }
            if (t_lb >= 0 && t_lb < ntiles && mbar_test_wait(&bars->lbd_st, n_lb & 1)) {
                const Tile x = tile_of(t_lb, p);
                st_release(p.lb_done + (int64_t)x.g * p.H + x.h, 1);
                LA_TRACE(t_lb, TR_LB_END);
                mbar_arrive(&bars->lbd_pub);
                ++n_lb; ++k_lb; t_lb = -1; any = true;
            }
            if (t_ag >= 0 && t_ag < ntiles && mbar_test_wait(&bars->agg_st[n_ag & 1], (n_ag >> 1) & 1)) {
                const Tile x = tile_of(t_ag, p);
                LA_TRACE(t_ag, TR_PUB_AGG);
                if (t_ag != p.suppress_tile) {
                    st_release(p.agg_flag + (int64_t)x.g * p.H + x.h, 1);
                    LA_TRACE(t_ag, TR_AGG);
                }
                ++n_ag; ++k_ag; t_ag = -1; any = true;
            }
            if (t_in >= 0 && t_in < ntiles && mbar_test_wait(&bars->incl_st, n_in & 1)) {
                const Tile x = tile_of(t_in, p);
                LA_TRACE(t_in, TR_PUB_INCL);
                if (t_in != p.suppress_tile) {
                    st_release(p.incl_flag + (int64_t)x.g * p.H + x.h, 1);
                    LA_TRACE(t_in, TR_INCL);
                }
                mbar_arrive(&bars->incl_pub);
                ++n_in; ++k_in; t_in = -1; any = true;
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
