// Lightning Attention prefill with the running state kept on chip: one
// persistent CTA per (sequence, head, half of the value columns), blocks of
// that sequence walked in order. bf16, d = 128, B in {128, 256}.
//
// Method (page "MiniMax-01 Lightning Attention", section "Lightning Attention
// 设计"; page "首个线性注意力架构的大模型来了…", section "4.1 创新的线性注意力",
// 双阶段计算):
//   O_b = (Q_b K_b^T, causal mask) V_b  +  Q_b . KV_b,
//   KV_0 = S0,  KV_{b+1} = KV_b + K_b^T V_b   (exclusive prefix over the blocks).
// Column j of O_b and of KV depends on column j of V only, so one (sequence,
// head) splits into two independent halves of 64 value columns. Each half is
// one work item; work items are taken round-robin by the CTAs, longest
// sequence first. Inside a work item the exclusive prefix is a running sum:
// the tensor cores accumulate K_b^T V_b into a fp32 TMEM accumulator block
// after block, and before block b's keys are added the state group copies
// KV_b (+ S0) out as the bf16 operand of the inter-block product. No block
// state ever goes to global memory, so Q, K, V are read once per work item
// and O is written once.
//
// A block of B rows is R = B/128 sub-units of 128 query rows; keys arrive in
// chunks of 128 (chunk j = keys 128j .. 128j+127 of the block). Items
// (chunk j, sub-unit r) with j <= r, in the order (0,0), (0,1), (1,1):
//   inter   O_r  = Q_r . bf16(KV_b)     (M=128, N=64,  K=128)  before sub-unit r's first PV
//   scores  S = Q_r K_j^T               (M=128, N=128, K=128)  -> TMEM
//   P       = bf16(mask(S)), written back into TMEM (two warpgroups, one per
//             64-key half of the chunk)
//   PV      O_r += P V_j                (M=128, N=64,  K=128)  A from TMEM
//   state   KV += K_j^T V_j             (M=128, N=64,  K=128)  as soon as chunk j is loaded
// This order retires shared-memory stages in ring order and early. K, V and
// Q have rings of their own, sized by how long a stage is held: a K chunk
// until its scores and state MMA (3 stages of 32 KB), a V chunk until its PVs
// and state MMA (2 of 16 KB), a Q sub-unit until its scores and inter-block
// MMA (2 of 32 KB); together they keep about one block of loads in flight.
// Roles (640 threads):
//   warp 0 (lane 0)  TMA producer of Q sub-units, K and V chunks: one
//                    non-blocking event loop over the three rings
//   warp 1 (lane 0)  tcgen05 issuer A: score MMAs and state MMAs (chunk by
//                    chunk as they land), a non-blocking event loop
//   warp 3 (lane 0)  tcgen05 issuer B: inter-block and PV MMAs, in item order
//                    Two issuing threads keep the tensor pipe fed while either
//                    one waits or does its bookkeeping; their MMAs are not
//                    ordered with each other, so every hand-off between them
//                    goes through an mbarrier (a score buffer is rewritten only
//                    after the PV that read it has completed).
//   warps 4-7, 8-11  scores -> P, keys 0-63 and 64-127 of every item
//   warps 12-15      state copy-out: TMEM fp32 -> bf16 shared operand (S0, when
//                    given, is stored into the accumulator at a work item's start)
//   warps 16-19      O epilogue: TMEM -> bf16 -> 16-byte stores of each row
//                    (masked for a ragged last sub-unit of a sequence)
// The instruction working set of the 20 warps is what limits the block rate
// once many SMs run the kernel (instruction fetch stalls grow with the number
// of SMs), so cold paths (finding the next work item, the waiting loop of a
// bounded wait, trace stamps) are out of line and the score masking has a
// single code path.
// Every wait is bounded (globaltimer); on expiry the CTA records
// LA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "sm100.cuh"
#include "pipe.cuh"
#include "decay.cuh"

namespace la {
namespace chain {

using namespace la::sm100;

constexpr int D = 128;                     // head dim (d_k = d_v)
constexpr int DV = 64;                     // value columns per work item
constexpr int UM = 128;                    // rows per sub-unit (MMA M)
constexpr int KC = 128;                    // keys per chunk
#ifndef LA_CHAIN_NQ
#define LA_CHAIN_NQ 2
#endif
#ifndef LA_CHAIN_NK
#define LA_CHAIN_NK 3
#endif
#ifndef LA_CHAIN_NV
#define LA_CHAIN_NV 2
#endif
constexpr int NQ = LA_CHAIN_NQ;            // Q sub-unit stages
constexpr int NK_MAX = LA_CHAIN_NK > 2 ? LA_CHAIN_NK : 2;   // K chunk stages, either instance
constexpr int NV_MAX = 3;                  // V chunk stages, either instance (barrier arrays)
constexpr int NS = 2;                      // score buffers in TMEM
constexpr int NTHREADS = 640;

constexpr uint32_t QH_BYTES = UM * 64 * 2;       // 16 KB: 128 rows x 64 columns
constexpr uint32_t Q_BYTES = 2 * QH_BYTES;       // 32 KB
constexpr uint32_t KH_BYTES = KC * 64 * 2;       // 16 KB: 128 keys x 64 columns
constexpr uint32_t K_BYTES = 2 * KH_BYTES;       // 32 KB
constexpr uint32_t V_BYTES = KC * DV * 2;        // 16 KB
constexpr uint32_t SB_BYTES = D * DV * 2;        // 16 KB: bf16 KV_b, 128 rows x 64 columns

// Shared-memory layout. The decay instance (a rate per head on the state) also
// keeps a ring of decay-weighted V chunks, the B operand of its state MMAs.
#ifndef LA_CHAIN_NVW
#define LA_CHAIN_NVW 2
#endif
#ifndef LA_CHAIN_DECAY_NV
#define LA_CHAIN_DECAY_NV 3
#endif
template <bool kDecay>
struct Smem {
    static constexpr int NK = kDecay && LA_CHAIN_NVW > 1 ? 2 : LA_CHAIN_NK;   // K chunk stages
    static constexpr int NV = kDecay ? LA_CHAIN_DECAY_NV : LA_CHAIN_NV;      // V chunk stages
    static constexpr int NVW = LA_CHAIN_NVW;                               // weighted V stages (decay only)
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + NQ * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + NK * K_BYTES;
    static constexpr uint32_t OFF_VW = OFF_V + NV * V_BYTES;               // weighted V (decay only)
    static constexpr uint32_t OFF_SB = OFF_VW + (kDecay ? NVW * V_BYTES : 0);
    static constexpr uint32_t OFF_BAR = OFF_SB + SB_BYTES;
    static constexpr uint32_t BYTES = OFF_BAR + 512 + 1024;   // + barriers + 1 KB alignment slack
    static_assert(BYTES <= 232448, "shared memory per CTA");
    static_assert(NK <= NK_MAX && NV <= NV_MAX && NVW <= NV_MAX, "barrier arrays");
};

// TMEM columns (512 x 32-bit, 128 lanes): three O slots, the state, NS score buffers.
constexpr uint32_t TM_O = 0, TM_KV = 192, TM_S = 256, TM_COLS = 512;
static_assert(TM_S + NS * KC <= TM_COLS, "TMEM budget");

constexpr uint32_t IDESC_S = idesc_bf16(UM, KC, false, false);   // Q (K-major) x K (K-major)
constexpr uint32_t IDESC_PV = idesc_bf16(UM, DV, false, true);   // P (TMEM) x V (MN-major)
constexpr uint32_t IDESC_KV = idesc_bf16(D, DV, true, true);     // K^T (MN-major) x V (MN-major)
constexpr uint32_t IDESC_C = idesc_bf16(UM, DV, false, true);    // Q (K-major) x KV (MN-major)

struct Bars {
    uint64_t q_full[NQ], q_empty[NQ];
    uint64_t k_full[NK_MAX], k_empty[NK_MAX]; // k_empty: two arrivals, the chunk's scores and its state MMA
    uint64_t v_full[NV_MAX], v_empty[NV_MAX]; // v_empty: the chunk's PVs and its state MMA (decay instance:
                                          // 1 + 128 arrivals, the PVs and the epilogue group that reads it
                                          // for the weighted copy)
    uint64_t vw_full[NV_MAX], vw_empty[NV_MAX]; // decay instance: weighted V chunk written / read by its state MMA
    uint64_t s_full[NS], p_full[NS], s_free[NS];
    uint64_t o_full[3], o_empty[3];
    uint64_t kv_ready;        // issuer -> state group: KV accumulator holds the next block's prefix
    uint64_t kv_read[4];      // state group -> issuer: accumulator read for block n (n % 4)
    uint64_t sb_full, sb_empty;
    uint64_t drain, drain_b;
    uint32_t tmem_base;
    int abort_flag;
    uint32_t peer_blocks;     // blocks whose Q and K loads the other CTA of the cluster has issued
};
static_assert(sizeof(Bars) <= 512, "barrier block");

// The two CTAs of a cluster walk the two value halves of the same work items (items 2c + k G
// and 2c + 1 + k G, G the even grid size), so they read the same Q and K tiles. A producer
// issues block n's Q and K loads only while the other is at most kPeerLag blocks behind,
// which keeps the second read of every tile in L2 over any number of blocks.
constexpr uint32_t kPeerLag = 2;
__device__ __forceinline__ uint32_t cluster_rank_of_cta() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Relaxed store to the same shared-memory variable of the other CTA of the pair.
__device__ __forceinline__ void st_peer_u32(const void* local, uint32_t value) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(cluster_rank_of_cta() ^ 1u));
    asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(a), "r"(value) : "memory");
}
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct Params {
    __nv_bfloat16* out;
    const SeqEntry* seqs;     // [nseq] first token and length
    const int32_t* order;     // [nseq] sequences, longest first
    const Control* ctrl;
    const float* init;        // [nseq][H][D][D] carried-in state, or nullptr
    float* state_out;         // [nseq][H][D][D] final states (the state-output instance only)
    const __nv_bfloat16* k;   // K and V, [T][H][D]: the few tokens of a ragged last chunk past its
    const __nv_bfloat16* v;   // last full 16-key MMA step (state-output instance only)
    const float* decay;       // [H] decay rates (the decay instance only)
    const __nv_bfloat16* q;   // Q [T][H][D]: the one-token sequences' queries (state-output instance only)
    int H, B, log2B, nseq;
    uint64_t wait_ns;
    long long suppress_item;  // test hook: this work item never hands over its second block's prefix (-1: none)
    uint64_t* trace;          // optional [gridDim.x][trace_blocks][kTraceEvents] clock64 stamps, or nullptr
    int trace_blocks;         // blocks per CTA the trace buffer holds
};

// Phase stamps of the optional per-block trace (la_debug_set_trace), in SM
// clock cycles (clock64), indexed by the CTA's block counter n.
enum TraceEvent {
    TR_Q0 = 0,         // producer: first Q sub-unit load of the block issued
    TR_KV0 = 1,        // producer: K chunk 0 load issued
    TR_KVL = 2,        // producer: last V chunk load issued
    TR_S0 = 3,         // issuer: first score MMA of the block issued
    TR_PV0 = 4,        // issuer: first PV MMA issued (its P was ready)
    TR_C0 = 5,         // issuer: inter-block MMA of sub-unit 0 issued
    TR_KVR = 6,        // issuer: last state MMA issued (kv_ready committed)
    TR_CL = 7,         // issuer: inter-block MMA of the last sub-unit issued
    TR_P0 = 8,         // P groups: P of the first item written
    TR_PL = 9,         // P groups: P of the last item written
    TR_XR = 10,        // state group: accumulator ready seen
    TR_SB = 11,        // state group: bf16 prefix handed over
    TR_E0 = 12,        // state group: first sub-unit accumulator complete
    TR_EL = 13,        // state group: last sub-unit accumulator complete
    TR_ST = 14,        // epilogue group: last O store of the block issued
    TR_PVL = 15,       // issuer: last PV MMA issued
    kTraceEvents = 16
};
// The stamps cost instruction-cache space in every role, so they are compiled
// only into trace builds (-DLA_CHAIN_TRACE); otherwise a trace buffer is ignored.
#ifdef LA_CHAIN_TRACE
#define LA_CTRACE(n, ev)                                                                                   \
    do {                                                                                                   \
        if (p.trace && (int)(n) < p.trace_blocks)                                                          \
            p.trace[((int64_t)blockIdx.x * p.trace_blocks + (n)) * kTraceEvents + (ev)] = clock64();       \
    } while (0)
#else
#define LA_CTRACE(n, ev) do {} while (0)
#endif

// The block a cursor is at: its work item (w, seq, h, the sequence's first
// token tok_s and length len) and, within it, block b with its first token,
// rows, sub-units Rb and whether its K^T V is needed by a later block (more).
// len = 0: no block left.
// first: the item's first block in walking order (block 0, or the last block when
// walking backwards).
struct Blk { int w, seq, h, tok_s, len, b, tok0, rows, Rb, more, first; };

// The block after `c` (the first block of the next work item with tokens,
// from w + step on, after the last block of one); with `first`, the CTA's first
// block. Out of line: every role's cursor shares this one copy.
// `nseq` counts the sequences walked; with `multi_only` (the prefill with final states)
// the one-token sequences, listed after the others, are left to singles_phase. With
// `rev` (the anti-causal instance) an item's blocks are walked from the last to the first.
__device__ __noinline__ Blk next_blk(Blk c, bool first, int step, int nseq, bool multi_only, bool rev,
                                     const Control* ctrl, const int32_t* order, const SeqEntry* seqs, int H,
                                     int log2B) {
    const int bs = 1 << log2B;
    int nb = (c.len + bs - 1) >> log2B;
    if (!first && (rev ? c.b > 0 : c.b + 1 < nb)) {
        c.b += rev ? -1 : 1;
    } else {
        const int nitems = 2 * (multi_only ? ctrl->nmulti : nseq) * H;   // 2 nseq H < 2^31
        int w = first ? c.w : c.w + step;
        c.len = 0;
        for (; w < nitems; w += step) {
            const unsigned pair = (unsigned)w >> 1;
            const int seq = order[pair / (unsigned)H];
            const SeqEntry e = seqs[seq];
            if (e.len > 0) {
                c.seq = seq;
                c.h = (int)(pair % (unsigned)H);
                c.tok_s = e.tok0;
                c.len = e.len;
                break;
            }
        }
        c.w = w;
        nb = (c.len + bs - 1) >> log2B;
        c.b = rev && nb > 0 ? nb - 1 : 0;
    }
    c.tok0 = c.tok_s + (c.b << log2B);
    c.rows = min(bs, c.len - (c.b << log2B));
    c.Rb = (c.rows + UM - 1) / UM;
    c.more = rev ? c.b > 0 : c.b + 1 < nb;
    c.first = rev ? c.b == nb - 1 : c.b == 0;
    return c;
}

// Walks this CTA's work items -> blocks -> items in the order every role uses,
// with the running counters that index the rings: n (blocks), q0 (Q
// sub-units), kc0 (K/V chunks), o0 (uses of O slot 0) at the current block,
// and i (items). A block has Rb = ceil(rows / 128) sub-units and as many
// 128-key chunks; its items are (0,0), (0,1), (1,1) when Rb = 2 and (0,0)
// when Rb = 1.
// kRev (the anti-causal instance): blocks walked backwards, items (0,0), (1,0), (1,1).
template <bool kRev>
struct CursorT {
    Blk bk;
    int w, seq, h, half, tok0, rows, Rb, b;
    bool add_state;                      // the block's K^T V is needed (not the last block)
    uint32_t n, q0, kc0, o0;
    int k;                               // item within the block
    int j, r;                            // its chunk and sub-unit
    uint32_t i;
    bool valid;

    __device__ __forceinline__ void set_item() {
        if (Rb == 2) {
            j = kRev ? (k == 0 ? 0 : 1) : (k == 2 ? 1 : 0);
            r = kRev ? (k == 2 ? 1 : 0) : (k == 0 ? 0 : 1);
        } else {
            j = 0;
            r = 0;
        }
    }
    __device__ __forceinline__ void take(const Params& p, bool first) {
        bk = next_blk(bk, first, gridDim.x, p.nseq, p.state_out != nullptr, kRev, p.ctrl, p.order, p.seqs, p.H,
                      p.log2B);
        valid = bk.len > 0;
        w = bk.w;
        seq = bk.seq;
        h = bk.h;
        half = bk.w & 1;
        tok0 = bk.tok0;
        rows = bk.rows;
        Rb = bk.Rb;
        b = bk.b;
        add_state = bk.more != 0;
        k = 0;
        set_item();
    }
    __device__ __forceinline__ void init(const Params& p) {
        n = q0 = kc0 = o0 = 0;
        i = 0;
        bk.w = blockIdx.x;
        bk.len = 0;
        bk.b = 0;
        if (p.ctrl->ok) take(p, true);
        else valid = false;
    }
    __device__ __forceinline__ void next_block(const Params& p) {
        ++n;
        q0 += Rb;
        kc0 += Rb;
        if (Rb == 2) ++o0;
        take(p, false);
    }
    __device__ __forceinline__ void next_item(const Params& p) {
        ++i;
        if (++k < (Rb == 2 ? 3 : 1)) {
            set_item();
            return;
        }
        next_block(p);
    }
    // item properties (forward: (0,0), (0,1), (1,1); anti-causal: (0,0), (1,0), (1,1))
    __device__ __forceinline__ bool first_of_chunk() const { return k != (kRev ? 2 : 1); }
    __device__ __forceinline__ bool last_of_chunk() const { return k != (kRev ? 1 : 0) || Rb == 1; }
    __device__ __forceinline__ bool first_of_sub() const { return kRev ? k != 1 : j == 0; }
    __device__ __forceinline__ bool last_of_sub() const { return k != (kRev ? 0 : 1) || Rb == 1; }
    __device__ __forceinline__ bool last_of_block() const { return k == (Rb == 2 ? 2 : 0); }
    // O slot of sub-unit rr: the sub-unit that finishes last alternates between
    // slots 1 and 2 from block to block; sub-unit 0 of a two-sub-unit block
    // (finished mid-block) always uses slot 0.
    __device__ __forceinline__ uint32_t oslot(int rr) const { return rr == Rb - 1 ? 1 + (n & 1) : 0; }
    __device__ __forceinline__ uint32_t ouse(int rr) const { return rr == Rb - 1 ? (n >> 1) : o0; }
};
using Cursor = CursorT<false>;

// Decay instance: the weighted copy lambda^(rows-1-c) v_c (c the key in the block, zero past the
// block's end) of every V chunk of the cursor's block, the B operand of its state MMAs, written by
// the 128 threads of the epilogue group; then their releases of the V chunk (the state MMA's share
// of v_empty). A chunk whose state MMA does not run passes through the ring unwritten. A line of
// the swizzled chunk is one key's 64 columns, so lines are scaled whole; 8 threads per line, each
// warp 4 lines (512 contiguous bytes) per step. Packed bf16 products: the weight is rounded to bf16
// and so is each product. Returns false when a wait gave up.
// (Out of line, taking the cursor's fields by value: the epilogue group calls it from two places,
// and the decay instance's block rate at 64 heads is set partly by instruction fetch.)
template <bool kStateOut, class SM>
__device__ __noinline__ bool weight_block_v(int h, int Rb, uint32_t kc0, bool add_state, int rows, const Params& p,
                                            Bars* bars, uint8_t* smem, int quad, int lane, volatile int* ab_cta,
                                            volatile int* ab_global, uint64_t ab_limit) {
    const Abort ab{ab_cta, ab_global, ab_limit};
    const float l2 = log2f(__ldg(p.decay + h));
    for (int j = 0; j < Rb; ++j) {
        const uint32_t kc = kc0 + j, st = kc % SM::NV, sw = kc % SM::NVW;
        if (!warp_all(wait_bar(&bars->v_full[st], (kc / SM::NV) & 1, ab)) ||
            !warp_all(wait_bar(&bars->vw_empty[sw], ((kc / SM::NVW) & 1) ^ 1, ab)))
            return false;
        if (add_state || kStateOut) {
            const uint8_t* src = smem + SM::OFF_V + st * V_BYTES;
            uint8_t* dst = smem + SM::OFF_VW + sw * V_BYTES;
#pragma unroll 2
            for (int it = 0; it < KC / 16; ++it) {
                const int line = 16 * it + 4 * quad + (lane >> 3);          // key KC*j + line
                const int t = KC * j + line;
                const __nv_bfloat162 w2 = __float2bfloat162_rn(t < rows ? decay_pow(l2, rows - 1 - t) : 0.f);
                const uint32_t off = line * 128 + (lane & 7) * 16;
                uint4 u = *reinterpret_cast<const uint4*>(src + off);
                __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                for (int x = 0; x < 4; ++x) e[x] = __hmul2(e[x], w2);
                *reinterpret_cast<uint4*>(dst + off) = u;
            }
            fence_proxy_async_smem();
        }
        mbar_arrive(&bars->vw_full[sw]);
        mbar_arrive(&bars->v_empty[st]);                 // done reading the V chunk
    }
    return true;
}
template <bool kStateOut, class SM>
__device__ __forceinline__ bool weight_block(const Cursor& c, const Params& p, Bars* bars, uint8_t* smem, int quad,
                                             int lane, const Abort& ab) {
    if (!c.valid) return true;
    return weight_block_v<kStateOut, SM>(c.h, c.Rb, c.kc0, c.add_state, c.rows, p, bars, smem, quad, lane, ab.cta,
                                         ab.global, ab.limit_ns);
}

// Anti-causal instance, the block walked after a sequence's ragged last block (walked first):
// that block's rows past the sequence end belong to the next sequence, so its state MMAs were
// skipped; its 1..B-1 tokens' k^T v (row m of the state, this CTA's 64 value columns) is added
// here on CUDA cores to what the accumulator holds (S0, seeded at the first block, or nothing),
// and written back for the later blocks' MMAs to add onto. Out of line: a cold path, once per
// sequence at most. Ends with the TMEM stores complete.
__device__ __noinline__ void rev_ragged_state(const Params& p, uint32_t tkv, int m, int tok_first, int tok_end,
                                              int h, int half) {
    if (p.init) tc_fence_after();
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {                     // one 32-column half at a time
        float x[32];
        if (p.init) {
            uint32_t a[32];
            tmem_ld_x32(tkv + 32 * hh, a);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) x[q] = __uint_as_float(a[q]);
        } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) x[q] = 0.f;
        }
        for (int t = tok_first; t < tok_end; ++t) {
            const float ki = __bfloat162float(p.k[((int64_t)t * p.H + h) * D + m]);
            const uint4* vr = reinterpret_cast<const uint4*>(p.v + ((int64_t)t * p.H + h) * D + DV * half + 32 * hh);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const uint4 u = __ldg(vr + g);
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * g + 2 * e] = fmaf(ki, __uint_as_float(w4[e] << 16), x[8 * g + 2 * e]);
                    x[8 * g + 2 * e + 1] = fmaf(ki, __uint_as_float(w4[e] & 0xffff0000u), x[8 * g + 2 * e + 1]);
                }
            }
        }
        uint32_t a[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) a[q] = __float_as_uint(x[q]);
        tmem_st_x32(tkv + 32 * hh, a);
    }
    tmem_wait_st();
}

// State-output instance, a work item's last block: row m of the final state (this CTA's 64
// value columns) = the accumulator (zero when no MMA ever ran: `none`) plus the tokens
// tok_first..tok_end-1 past the last full 16-key MMA step, on CUDA cores (with decay each
// weighted by lambda^(tok_end - 1 - t)), stored to state_out. Out of line and a 32-column half
// at a time, so it adds no register pressure to the pipeline roles.
template <bool kDecay>
__device__ __noinline__ void write_final_state(const Params& p, uint32_t tkv, int m, bool none, int tok_first,
                                               int tok_end, int seq, int h, int half) {
    float* row = p.state_out + (((int64_t)seq * p.H + h) * D + m) * D + DV * half;
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
        float x[32];
        uint32_t a[32];
        tmem_ld_x32(tkv + 32 * hh, a);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) x[q] = none ? 0.f : __uint_as_float(a[q]);
        for (int t = tok_first; t < tok_end; ++t) {
            float ki = __bfloat162float(p.k[((int64_t)t * p.H + h) * D + m]);
            if constexpr (kDecay) ki *= decay_pow(log2f(__ldg(p.decay + h)), tok_end - 1 - t);
            const uint4* vr = reinterpret_cast<const uint4*>(p.v + ((int64_t)t * p.H + h) * D + DV * half + 32 * hh);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const uint4 u = __ldg(vr + g);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * g + 2 * e] += ki * __uint_as_float(w[e] << 16);
                    x[8 * g + 2 * e + 1] += ki * __uint_as_float(w[e] & 0xffff0000u);
                }
            }
        }
        float4* dst = reinterpret_cast<float4*>(row + 32 * hh);
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
    }
}

// State-output instance, after the CTA's chain work: the one-token sequences of the batch
// (a serving batch's continuations, each with its carried-in state) are one recurrent
// step each, the decode step's arithmetic at HBM rate instead of a chain work item:
//   S = lambda S0 + k^T v,  o = lambda (q S0) + (q . k) v   (lambda = 1 without decay),
// with the new state written to state_out (which may be init itself). (Sequence, head)
// pairs are taken by atomic ticket, so the CTAs that finish their chain items first take
// more of them. With one CTA per SM the bytes in flight come from bulk copies: warp 0
// (lane 0) streams each pair's 64 KB S0 and its q, k, v rows into a ring of three
// shared-memory slots (cp.async.bulk, completing on the slot's barrier) and writes each
// updated slot back to state_out with a bulk store; warps 4-19 (512 threads: 32 column
// groups of 16 bytes x 16 row groups, 8 rows each) update the slot in place and form o.
// (Stores from registers instead of the bulk store measured 10% slower.) The shared
// memory of the finished pipeline is reused; every wait is bounded.
constexpr int kSingleSlots = 3;
constexpr int kTicketChunk = 32;                                           // pairs taken per ticket
constexpr uint32_t SS_STATE = D * D * 4;                                    // 64 KB
constexpr uint32_t SS_QKV = kSingleSlots * SS_STATE;                       // q, k, v rows: 768 B a slot
constexpr uint32_t SS_META = SS_QKV + kSingleSlots * 768;                  // per slot: pair, head, o row, state offset
constexpr uint32_t SS_CHUNK = SS_META + kSingleSlots * 32;                 // the current ticket chunk's pairs
constexpr uint32_t SS_RED = SS_CHUNK + kTicketChunk * 32;                  // [16][32] float4 partial q S0
constexpr uint32_t SS_QK = SS_RED + 16 * 32 * 16;                          // [16] partial q . k
constexpr uint32_t SS_BAR = SS_QK + 16 * 4;                                // full[3], done[3]
constexpr uint32_t SS_END = SS_BAR + 2 * kSingleSlots * 8;
static_assert(SS_END <= Smem<false>::OFF_BAR && SS_END <= Smem<true>::OFF_BAR, "one-token phase fits before the barriers");

// one (sequence, head) of the phase: ticket t, head h, its token's row offset in Q, K, V, O,
// and the offset of its d x d state
struct SinglePair { int32_t t, h; int64_t row, sbase; };
static_assert(sizeof(SinglePair) == 24, "pair record");

template <bool kDecay>
__device__ __noinline__ void singles_phase(const Params& p, uint8_t* smem, const Abort ab) {
    constexpr int CG = D / 4, RG = 16, ROWS = D / RG;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SS_BAR);
    uint64_t* done = full + kSingleSlots;
    SinglePair* meta = reinterpret_cast<SinglePair*>(smem + SS_META);      // stride 32 bytes: meta[b] at 32 b
    SinglePair* chunk = reinterpret_cast<SinglePair*>(smem + SS_CHUNK);    // stride 32 bytes
    float4* red = reinterpret_cast<float4*>(smem + SS_RED);
    float* qkp = reinterpret_cast<float*>(smem + SS_QK);
    auto slot_meta = [&](uint32_t b) -> volatile SinglePair& {
        return *reinterpret_cast<volatile SinglePair*>(reinterpret_cast<uint8_t*>(meta) + 32 * b);
    };
    Control* ctrl = const_cast<Control*>(p.ctrl);
    const int nmulti = ctrl->nmulti;
    const int64_t npairs = (int64_t)ctrl->nsingle * p.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int b = 0; b < kSingleSlots; ++b) { mbar_init(&full[b], 1); mbar_init(&done[b], 1); }
    }
    __syncthreads();
    if (warp == 0) {
        // ---------------------------------------------------------------- bulk copies (warp 0)
        // The warp takes kTicketChunk pairs per ticket and looks their sequences up in
        // parallel; lane 0 issues every copy and store (its bulk groups), the warp's
        // decisions are uniform.
        const uint32_t state_bytes = p.init ? SS_STATE : 0u;
        const uint64_t once = policy_evict_first();   // every state is streamed through once
        uint32_t L = 0, S = 0;                   // pairs loaded, pairs stored (slot = count % 3)
        int c_len = 0, c_pos = 0;
        bool end = false, ok = true;
        uint32_t idle = 0;
        uint64_t t_idle = 0;
        while (ok && !(end && S == L)) {
            bool prog = false;
            if (!end && L - S < (uint32_t)kSingleSlots) {
                if (c_pos == c_len) {
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&ctrl->ticket, kTicketChunk);
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const int64_t t = (int64_t)base + lane;
                    if (t < npairs) {
                        const int seq = p.order[nmulti + (int)(t / p.H)], h = (int)(t % p.H);
                        SinglePair& e = *reinterpret_cast<SinglePair*>(reinterpret_cast<uint8_t*>(chunk) + 32 * lane);
                        e.t = (int32_t)t;
                        e.h = h;
                        e.row = ((int64_t)p.seqs[seq].tok0 * p.H + h) * D;
                        e.sbase = ((int64_t)seq * p.H + h) * D * D;
                    }
                    __syncwarp();
                    const int64_t left = npairs - base;
                    c_len = left <= 0 ? 0 : (left < kTicketChunk ? (int)left : kTicketChunk);
                    c_pos = 0;
                }
                const uint32_t b = L % kSingleSlots;
                if (c_len == 0) {
                    if (lane == 0) {
                        slot_meta(b).t = -1;         // the compute threads stop at this slot
                        mbar_arrive(&full[b]);
                    }
                    end = true;
                } else {
                    if (lane == 0) {
                        // the store of this slot's previous pair (L - 3) must have read the slot
                        if (L >= (uint32_t)kSingleSlots) {
                            const uint32_t later = S - (L - kSingleSlots) - 1;   // stores issued after it
                            if (later == 0) bulk_wait_read0(); else if (later == 1) bulk_wait_read1(); else bulk_wait_read2();
                        }
                        const SinglePair e = *reinterpret_cast<const SinglePair*>(reinterpret_cast<uint8_t*>(chunk) + 32 * c_pos);
                        volatile SinglePair& m = slot_meta(b);
                        m.t = e.t; m.h = e.h; m.row = e.row; m.sbase = e.sbase;
                        uint8_t* qkv = smem + SS_QKV + b * 768;
                        mbar_expect_tx(&full[b], 768 + state_bytes);
                        if (state_bytes) bulk_load_hint(smem + b * SS_STATE, p.init + e.sbase, SS_STATE, &full[b], once);
                        bulk_load(qkv, p.q + e.row, 256, &full[b]);
                        bulk_load(qkv + 256, p.k + e.row, 256, &full[b]);
                        bulk_load(qkv + 512, p.v + e.row, 256, &full[b]);
                    }
                    ++c_pos;
                    ++L;
                }
                prog = true;
            }
            if (S < L) {                         // the oldest slot in use has been computed: store it
                int rdy = 0;
                if (lane == 0) rdy = mbar_test_wait(&done[S % kSingleSlots], (S / kSingleSlots) & 1);
                if (__shfl_sync(0xffffffffu, rdy, 0)) {
                    if (lane == 0) {
                        const uint32_t b = S % kSingleSlots;
                        bulk_store_hint(p.state_out + slot_meta(b).sbase, smem + b * SS_STATE, SS_STATE, once);
                        bulk_commit();
                    }
                    ++S;
                    prog = true;
                }
            }
            if (prog) {
                idle = 0;
            } else if ((++idle & 63u) == 0) {
                int stop = 0;
                if (lane == 0) {
                    if (ab.raised()) { *ab.cta = 1; stop = 1; }
                    else {
                        const uint64_t now = globaltimer_ns();
                        if (idle == 64) t_idle = now;
                        else if (now - t_idle > ab.limit_ns) { ab.raise(); stop = 1; }
                    }
                }
                if (__shfl_sync(0xffffffffu, stop, 0)) ok = false;
            }
        }
        if (lane == 0) bulk_wait0();            // every store complete before the CTA ends
    } else if (threadIdx.x >= 128) {
        // ---------------------------------------------------------------- state update
        // Named barrier 1 over these 512 threads. A thread whose wait ran out (the launch is
        // aborting) still passes every barrier of the iteration, and the exit is decided for
        // all of them at once (bar.red.or), so no thread waits on one that has left.
        const int ct = threadIdx.x - 128, cg = ct % CG, rg = ct / CG;
        for (uint32_t k = 0;; ++k) {
            const uint32_t b = k % kSingleSlots;
            const bool got = warp_all(wait_bar(&full[b], (k / kSingleSlots) & 1, ab));
            const volatile SinglePair& m = slot_meta(b);
            const bool stop = !got || m.t < 0;
            if (!stop) {
                const int h = m.h;
                float lam = 1.f;
                if constexpr (kDecay) lam = __ldg(p.decay + h);
                const __nv_bfloat16* qkv = reinterpret_cast<const __nv_bfloat16*>(smem + SS_QKV + b * 768);
                float4* Sm = reinterpret_cast<float4*>(smem + b * SS_STATE);
                const float4 vv = make_float4(__bfloat162float(qkv[256 + 4 * cg]), __bfloat162float(qkv[257 + 4 * cg]),
                                              __bfloat162float(qkv[258 + 4 * cg]), __bfloat162float(qkv[259 + 4 * cg]));
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                float qk = 0.f;
#pragma unroll
                for (int a = 0; a < ROWS; ++a) {
                    const int i = rg + a * RG;
                    const float qi = __bfloat162float(qkv[i]), ki = __bfloat162float(qkv[128 + i]);
                    qk = fmaf(qi, ki, qk);
                    float4 x = p.init ? Sm[i * CG + cg] : make_float4(0.f, 0.f, 0.f, 0.f);
                    acc.x = fmaf(qi, x.x, acc.x); acc.y = fmaf(qi, x.y, acc.y);
                    acc.z = fmaf(qi, x.z, acc.z); acc.w = fmaf(qi, x.w, acc.w);
                    x.x = fmaf(ki, vv.x, lam * x.x); x.y = fmaf(ki, vv.y, lam * x.y);
                    x.z = fmaf(ki, vv.z, lam * x.z); x.w = fmaf(ki, vv.w, lam * x.w);
                    Sm[i * CG + cg] = x;
                }
                red[rg * CG + cg] = acc;
                if (cg == 0) qkp[rg] = qk;           // q . k over this row group's rows
                fence_proxy_async_smem();            // this thread's slot writes, before the bulk store reads them
            }
            bar_named(1, 512);
            if (!stop && ct < D) {
                const __nv_bfloat16* qkv = reinterpret_cast<const __nv_bfloat16*>(smem + SS_QKV + b * 768);
                float qkt = 0.f, sum = 0.f;
                const int c = ct / 4, l4 = ct % 4;
#pragma unroll
                for (int r = 0; r < RG; ++r) {
                    qkt += qkp[r];
                    const float4 x = red[r * CG + c];
                    sum += l4 == 0 ? x.x : l4 == 1 ? x.y : l4 == 2 ? x.z : x.w;
                }
                float lam = 1.f;
                if constexpr (kDecay) lam = __ldg(p.decay + m.h);
                p.out[m.row + ct] = __float2bfloat16_rn(fmaf(qkt, __bfloat162float(qkv[256 + ct]), lam * sum));
            }
            // the slot is complete and the reduction buffers may be rewritten; stop together
            if (bar_red_or(1, 512, stop)) break;
            if (ct == 0) mbar_arrive(&done[b]);
        }
    }
}

// kStateOut: also write each sequence's final state S0 + sum_t k_t^T v_t to
// p.state_out (the last block runs its state MMAs too; the copy-out group reads
// the accumulator after them). A separate instance, so the plain prefill's code
// is unchanged.
//
// kDecay: a decay rate lambda_h in [0, 1] per head on the state (decay.cuh):
// S_t = lambda S_{t-1} + k_t^T v_t. For a block of n rows, row r (in the block)
// and key c (in the block):
//   P[r][c]   = lambda^(r-c) S[r][c]                 (P groups, c <= r)
//   O_r       = (lambda^(r+1) q_r) bf16(KV_b) + ...  (the P groups write the
//               scaled Q row into the score buffer's columns that P leaves
//               free; the inter-block MMA reads its A operand from there)
//   KV_{b+1}  = lambda^n KV_b + sum_c K_c^T (lambda^(n-1-c) v_c)
//               (copy-out group rescales the accumulator when it reads KV_b;
//               the epilogue group writes the weighted V chunks, the state
//               MMA's B operand, one block ahead)
// The weighted V and the scaled Q rows are packed bf16 products (weight and
// product each rounded to bf16: relative 2^-8 per term). Rates are checked
// before the launch (a bad rate leaves the launch with no work).
// kRev: the anti-causal instance (no state output, no decay), O_t = q_t S0 + sum_{s >= t,
// same sequence} (q_t . k_s) v_s: blocks walked from each sequence's end, the mask keeping
// keys at or after the query row, and the running state the suffix of the blocks walked.
// If the first block walked (the sequence's last) is ragged, its state is added on CUDA
// cores by the copy-out group at the next block (the rows past the sequence end belong to
// the next sequence, so no MMA may take them); its own state MMAs are skipped.
template <bool kStateOut, bool kDecay, bool kRev = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
prefill_chain_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Params p) {
    static_assert(!kRev || (!kStateOut && !kDecay), "the anti-causal instance has neither state output nor decay");
    using SM = Smem<kDecay>;
    using Cursor = CursorT<kRev>;
    constexpr int NK = SM::NK, NV = SM::NV;
    constexpr uint32_t OFF_Q = SM::OFF_Q, OFF_K = SM::OFF_K, OFF_V = SM::OFF_V, OFF_SB = SM::OFF_SB,
                       OFF_BAR = SM::OFF_BAR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Abort ab{&bars->abort_flag, const_cast<volatile int*>(&p.ctrl->abort), p.wait_ns};

    if (threadIdx.x == 0) {
        for (int i = 0; i < NQ; ++i) { mbar_init(&bars->q_full[i], 1); mbar_init(&bars->q_empty[i], 2); }
        for (int i = 0; i < NK; ++i) { mbar_init(&bars->k_full[i], 1); mbar_init(&bars->k_empty[i], 2); }
        // v_empty: the PVs' commit, then the state MMA's commit (the epilogue group's 128 threads,
        // which read V for the weighted copy, in the decay instance)
        for (int i = 0; i < NV; ++i) { mbar_init(&bars->v_full[i], 1); mbar_init(&bars->v_empty[i], kDecay ? 129 : 2); }
        for (int i = 0; i < NS; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 256);
            mbar_init(&bars->s_free[i], 1);
        }
        for (int i = 0; i < 3; ++i) { mbar_init(&bars->o_full[i], 1); mbar_init(&bars->o_empty[i], 128); }
        mbar_init(&bars->kv_ready, 1);
        for (int i = 0; i < 4; ++i) mbar_init(&bars->kv_read[i], 128);
        mbar_init(&bars->sb_full, 128);
        mbar_init(&bars->sb_empty, 1);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->drain_b, 1);
        if constexpr (kDecay) {
            for (int i = 0; i < SM::NVW; ++i) { mbar_init(&bars->vw_full[i], 128); mbar_init(&bars->vw_empty[i], 1); }
        }
        bars->abort_flag = 0;
        bars->peer_blocks = 0;
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
    cluster_barrier();            // both CTAs' barriers and progress words exist before any remote store
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ================================================================ TMA producer (Q, K, V)
        // One thread, three streams in a non-blocking event loop: each issues its next
        // load as soon as that load's stage is free, so no stream waits behind another.
        if (lane == 0) {
            const uint64_t once = policy_evict_first();      // V: read by this CTA only
            Cursor cq, ck, cv;
            cq.init(p);
            ck.init(p);
            cv.init(p);
            int rq = 0, rk = 0, rv = 0;                      // sub-unit / chunk within each stream's block
            uint32_t k_issued = 0, v_issued = 0, q_issued = 0;   // loads issued (ring indices)
            bool ok = true;
            uint32_t idle = 0;
            uint64_t t_idle = 0;
            uint32_t published = 0;                          // blocks whose Q and K loads are all issued
            const volatile uint32_t* peer = &bars->peer_blocks;
            while (cq.valid || ck.valid || cv.valid) {
                bool prog = false;
                const uint32_t lead = *peer + kPeerLag;      // highest block this CTA may load Q / K for
                if (cq.valid && cq.n <= lead) {
                    const uint32_t qc = cq.q0 + rq;
                    if (mbar_test_wait(&bars->q_empty[qc % NQ], ((qc / NQ) & 1) ^ 1)) {
                        const int t = cq.tok0 + UM * rq;
                        uint8_t* qd = smem + OFF_Q + (qc % NQ) * Q_BYTES;
                        mbar_expect_tx(&bars->q_full[qc % NQ], Q_BYTES);
                        tma_load_3d(qd, &tmQ, &bars->q_full[qc % NQ], 0, cq.h, t);
                        tma_load_3d(qd + QH_BYTES, &tmQ, &bars->q_full[qc % NQ], 64, cq.h, t);
                        q_issued = qc + 1;
                        if (rq == 0) LA_CTRACE(cq.n, TR_Q0);
                        if (++rq == cq.Rb) { rq = 0; cq.next_block(p); }
                        prog = true;
                    }
                }
                if (ck.valid && ck.n <= lead) {
                    const uint32_t kc = ck.kc0 + rk;
                    if (mbar_test_wait(&bars->k_empty[kc % NK], ((kc / NK) & 1) ^ 1)) {
                        const int t = ck.tok0 + KC * rk;
                        uint8_t* kd = smem + OFF_K + (kc % NK) * K_BYTES;
                        mbar_expect_tx(&bars->k_full[kc % NK], K_BYTES);
                        tma_load_3d(kd, &tmK, &bars->k_full[kc % NK], 0, ck.h, t);
                        tma_load_3d(kd + KH_BYTES, &tmK, &bars->k_full[kc % NK], 64, ck.h, t);
                        k_issued = kc + 1;
                        if (rk == 0) LA_CTRACE(ck.n, TR_KV0);
                        if (++rk == ck.Rb) { rk = 0; ck.next_block(p); }
                        prog = true;
                    }
                }
                if (cv.valid) {
                    const uint32_t kc = cv.kc0 + rv;
                    if (mbar_test_wait(&bars->v_empty[kc % NV], ((kc / NV) & 1) ^ 1)) {
                        const int t = cv.tok0 + KC * rv;
                        mbar_expect_tx(&bars->v_full[kc % NV], V_BYTES);
                        tma_load_3d_hint(smem + OFF_V + (kc % NV) * V_BYTES, &tmV, &bars->v_full[kc % NV],
                                         DV * cv.half, cv.h, t, once);
                        v_issued = kc + 1;
                        if (rv == cv.Rb - 1) LA_CTRACE(cv.n, TR_KVL);
                        if (++rv == cv.Rb) { rv = 0; cv.next_block(p); }
                        prog = true;
                    }
                }
                // a cursor's block count stops at its total once the stream is done
                if (min(cq.n, ck.n) != published) {
                    published = min(cq.n, ck.n);
                    st_peer_u32(&bars->peer_blocks, published);
                }
                if (prog) {
                    idle = 0;
                } else if ((++idle & 63u) == 0) {
                    if (ab.raised()) { *ab.cta = 1; ok = false; break; }
                    const uint64_t now = globaltimer_ns();
                    if (idle == 64) t_idle = now;
                    else if (now - t_idle > ab.limit_ns) { ab.raise(); ok = false; break; }
                }
            }
            // let the other CTA run on freely from here (this CTA issues no more loads)
            st_peer_u32(&bars->peer_blocks, 0x7fffffffu);
            // On abort, wait (bounded) for this producer's copies still in flight
            // into shared memory: only the latest load of each stage can be pending.
            if (!ok) {
                auto drain = [&](uint64_t* full, uint32_t issued, uint32_t nst) {
                    for (uint32_t i = (issued > nst ? issued - nst : 0); i < issued; ++i) {
                        const uint64_t t0 = globaltimer_ns();
                        while (!mbar_try_wait(&full[i % nst], (i / nst) & 1) && globaltimer_ns() - t0 < 100000000ull) {}
                    }
                };
                drain(bars->q_full, q_issued, NQ);
                drain(bars->k_full, k_issued, NK);
                drain(bars->v_full, v_issued, NV);
            }
        }
    } else if (warp == 1 || warp == 3) {
        // Shared-memory descriptors: the base of each region once, then a 16-byte-unit
        // offset per operand step (the address field is the low 14 bits).
        const uint64_t dq = sdesc_sw128(smem_u32(smem + OFF_Q), 16, 1024);             // K-major
        const uint64_t dk = sdesc_sw128(smem_u32(smem + OFF_K), 16, 1024);             // K-major (scores)
        const uint64_t dkt = sdesc_sw128(smem_u32(smem + OFF_K), KH_BYTES, 1024);      // MN-major (state)
        const uint64_t dv = sdesc_sw128(smem_u32(smem + OFF_V), V_BYTES, 1024);
        const uint64_t dsb = sdesc_sw128(smem_u32(smem + OFF_SB), SB_BYTES, 1024);
        const uint64_t dvs = kDecay ? sdesc_sw128(smem_u32(smem + SM::OFF_VW), V_BYTES, 1024) : dv;   // state MMA's V
        if (warp == 1 && lane == 0) {
            // ============================================================ issuer A: scores, state MMAs
            // Event loop over two cursors; every step is taken only when its inputs are
            // ready (non-blocking mbarrier tests). The score cursor needs its score buffer
            // back (the PV that read it completed), its K chunk and, for a sub-unit's first
            // item, its Q rows. The state cursor follows it: chunk j's state MMA once the V
            // chunk is loaded and, for the block's first chunk, the state group has copied
            // the previous prefix out.
            Cursor sc, dc;
            sc.init(p);
            dc.init(p);
            uint32_t s_issued = 0;
            uint32_t kvr_blk = 0xffffffffu;       // block whose state copy-out has been seen
            uint32_t idle = 0;
            uint64_t t_idle = 0;
            while (sc.valid || dc.valid) {
                bool prog = false;
                if (sc.valid) {
                    const uint32_t kc = sc.kc0 + sc.j, qc = sc.q0 + sc.r, sbuf = sc.i % NS;
                    if ((sc.i < NS || mbar_test_wait(&bars->s_free[sbuf], ((sc.i / NS) - 1) & 1)) &&
                        (!sc.first_of_chunk() || mbar_test_wait(&bars->k_full[kc % NK], (kc / NK) & 1)) &&
                        (!sc.first_of_sub() || mbar_test_wait(&bars->q_full[qc % NQ], (qc / NQ) & 1))) {
                        tc_fence_after();
                        const uint64_t a = dq + (((qc % NQ) * Q_BYTES) >> 4), b = dk + (((kc % NK) * K_BYTES) >> 4);
                        const uint32_t d_s = tmem + TM_S + sbuf * KC;
#pragma unroll
                        for (int s = 0; s < D / 16; ++s)
                            mma_ss(d_s, a + (((s >> 2) * QH_BYTES + (s & 3) * 32) >> 4),
                                   b + (((s >> 2) * KH_BYTES + (s & 3) * 32) >> 4), IDESC_S, s > 0);
                        tc_commit(&bars->s_full[sbuf]);
                        if (sc.last_of_chunk()) tc_commit(&bars->k_empty[kc % NK]);   // the scores' share
                        if (sc.last_of_sub()) tc_commit(&bars->q_empty[qc % NQ]);     // the scores' share
                        ++s_issued;
                        if (sc.k == 0) LA_CTRACE(sc.n, TR_S0);
                        sc.next_item(p);
                        prog = true;
                    }
                }
                if (dc.valid && dc.i < s_issued) {
                    if (!dc.last_of_chunk()) {
                        dc.next_item(p);
                    } else {
                        const uint32_t kc = dc.kc0 + dc.j;
                        bool ready = kDecay ? mbar_test_wait(&bars->vw_full[kc % SM::NVW], (kc / SM::NVW) & 1)
                                            : mbar_test_wait(&bars->v_full[kc % NV], (kc / NV) & 1);
                        // the state MMAs of a block wait for the copy-out group to have read the
                        // prefix (and, with decay, rescaled it) whenever they run: in the
                        // state-output instance also on a sequence's last block
                        // the anti-causal instance's ragged first block: state added on CUDA cores
                        const bool run = (dc.add_state || kStateOut) &&
                                         !(kRev && dc.bk.first && dc.rows < (1 << p.log2B));
                        if (ready && run && dc.j == 0 && kvr_blk != dc.n) {
                            if (mbar_test_wait(&bars->kv_read[dc.n & 3], (dc.n >> 2) & 1)) kvr_blk = dc.n;
                            else ready = false;
                        }
                        if (ready) {
                            if (run) {
                                tc_fence_after();
                                const uint64_t a = dkt + (((kc % NK) * K_BYTES) >> 4),
                                               b = kDecay ? dvs + (((kc % SM::NVW) * V_BYTES) >> 4)
                                                          : dv + (((kc % NV) * V_BYTES) >> 4);
                                // a ragged last chunk: its full 16-key steps only (the copy-out
                                // group adds the rest); the rows past the sequence end belong to
                                // the next sequence
                                const int nsteps = dc.add_state ? KC / 16 : min(KC, dc.rows - KC * dc.j) >> 4;
#pragma unroll
                                for (int s = 0; s < KC / 16; ++s)
                                    if (s < nsteps)
                                        mma_ss(tmem + TM_KV, a + ((s * 2048) >> 4), b + ((s * 2048) >> 4), IDESC_KV,
                                               (!dc.bk.first || dc.j > 0 || s > 0 || p.init != nullptr));
                                if (dc.j == dc.Rb - 1) {
                                    tc_commit(&bars->kv_ready);
                                    LA_CTRACE(dc.n, TR_KVR);
                                }
                            }
                            tc_commit(&bars->k_empty[kc % NK]);          // the state MMA's shares
                            tc_commit(kDecay ? &bars->vw_empty[kc % SM::NVW] : &bars->v_empty[kc % NV]);
                            dc.next_item(p);
                            prog = true;
                        }
                    }
                }
                // ---- nothing ready: bounded idle time, launch-wide abort
                if (prog) {
                    idle = 0;
                } else if ((++idle & 63u) == 0) {
                    if (ab.raised()) { *ab.cta = 1; break; }
                    const uint64_t now = globaltimer_ns();
                    if (idle == 64) t_idle = now;
                    else if (now - t_idle > ab.limit_ns) { ab.raise(); break; }
                }
            }
            // every MMA issued by this thread has completed once `drain` fires
            tc_commit(&bars->drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars->drain, 0) && globaltimer_ns() - t0 < 1000000000ull) {}
        } else if (warp == 3 && lane == 0) {
            // ============================================================ issuer B: inter-block, PV
            // Item by item: the inter-block MMA first for a sub-unit's first item (it
            // initialises the accumulator), then the PV once the P groups have written P.
            Cursor c;
            c.init(p);
            bool ok = true;
            while (ok && c.valid) {
                const uint32_t sbuf = c.i % NS, slot = c.oslot(c.r);
                const uint32_t kc = c.kc0 + c.j, qc = c.q0 + c.r;
                const uint32_t d_o = tmem + TM_O + slot * 64;
                if (kDecay && c.first_of_sub()) {
                    // O_r = (Lambda Q_r) . bf16(KV_b) from TMEM: the P groups wrote lambda^(r+1) q_r
                    // (bf16) into the score buffer's columns that P leaves free
                    if (!wait_bar(&bars->o_empty[slot], (c.ouse(c.r) & 1) ^ 1, ab)) { ok = false; break; }
                    if (c.r == 0 && !wait_bar(&bars->sb_full, c.n & 1, ab)) { ok = false; break; }
                    if (!wait_bar(&bars->p_full[sbuf], (c.i / NS) & 1, ab)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_q = tmem + TM_S + sbuf * KC + 32;
#pragma unroll
                    for (int s = 0; s < D / 16; ++s)
                        mma_ts(d_o, a_q + (s < 4 ? s * 8 : 64 + (s - 4) * 8), dsb + ((s * 2048) >> 4), IDESC_PV,
                               s > 0);
                    if (c.r == c.Rb - 1) tc_commit(&bars->sb_empty);
                    tc_commit(&bars->q_empty[qc % NQ]);                  // the inter-block share (P groups read Q)
                    LA_CTRACE(c.n, c.r == 0 ? TR_C0 : TR_CL);
                } else if (c.first_of_sub()) {
                    // O_r = Q_r . bf16(KV_b)
                    if (!wait_bar(&bars->o_empty[slot], (c.ouse(c.r) & 1) ^ 1, ab)) { ok = false; break; }
                    if (c.r == 0 && !wait_bar(&bars->sb_full, c.n & 1, ab)) { ok = false; break; }
                    if (!wait_bar(&bars->q_full[qc % NQ], (qc / NQ) & 1, ab)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t a = dq + (((qc % NQ) * Q_BYTES) >> 4);
#pragma unroll
                    for (int s = 0; s < D / 16; ++s)
                        mma_ss(d_o, a + (((s >> 2) * QH_BYTES + (s & 3) * 32) >> 4), dsb + ((s * 2048) >> 4), IDESC_C,
                               s > 0);
                    if (c.r == c.Rb - 1) tc_commit(&bars->sb_empty);
                    tc_commit(&bars->q_empty[qc % NQ]);                  // the inter-block MMA's share
                    LA_CTRACE(c.n, c.r == 0 ? TR_C0 : TR_CL);
                }
                // O_r += P V_j; P of keys 0-63 in columns 0-31, of keys 64-127 in 64-95
                if (!wait_bar(&bars->p_full[sbuf], (c.i / NS) & 1, ab)) { ok = false; break; }
                if (c.first_of_chunk() && !wait_bar(&bars->v_full[kc % NV], (kc / NV) & 1, ab)) { ok = false; break; }
                tc_fence_after();
                const uint64_t b = dv + (((kc % NV) * V_BYTES) >> 4);
                const uint32_t a_p = tmem + TM_S + sbuf * KC;
#pragma unroll
                for (int s = 0; s < KC / 16; ++s)
                    mma_ts(d_o, a_p + (s < 4 ? s * 8 : 64 + (s - 4) * 8), b + ((s * 2048) >> 4), IDESC_PV, 1);
                tc_commit(&bars->s_free[sbuf]);
                if (c.last_of_chunk()) tc_commit(&bars->v_empty[kc % NV]);   // the PVs' share
                if (c.last_of_sub()) tc_commit(&bars->o_full[slot]);
                if (c.k == 0) LA_CTRACE(c.n, TR_PV0);
                if (c.last_of_block()) LA_CTRACE(c.n, TR_PVL);
                c.next_item(p);
            }
            tc_commit(&bars->drain_b);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bars->drain_b, 0) && globaltimer_ns() - t0 < 1000000000ull) {}
        }
    } else if (warp >= 4 && warp < 12) {
        // ================================================================ scores -> P
        const int hk = warp >= 8 ? 1 : 0;                // keys 0-63 or 64-127 of the chunk
        const int quad = warp & 3;
        const int m = quad * 32 + lane;                  // query row of the sub-unit (TMEM lane)
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        bool ok = true;
        Cursor c;
        c.init(p);
        while (ok && c.valid) {
            const uint32_t sbuf = c.i % NS;
            if (!warp_all(wait_bar(&bars->s_full[sbuf], (c.i / NS) & 1, ab))) { ok = false; break; }
            tc_fence_after();
            const uint32_t ts = tmem + lane_base + TM_S + sbuf * KC + 64 * hk;
            const int lim = UM * (c.r - c.j) + m - 64 * hk;    // key column kept when col <= lim
            float lam = 1.f, l2 = 0.f;
            if constexpr (kDecay) {
                lam = __ldg(p.decay + c.h);
                l2 = log2f(lam);
            }
            // P of these 64 keys goes over the first 32 of their columns, each 32-key half stored as
            // soon as it is packed: the store overlaps the next half's load, and 16 packed words are
            // live instead of 32. (Kept unrolled in every instance: rolled in the decay instance it
            // measured 7% slower.)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t a[32], ph[16];
                tmem_ld_x32(ts + 32 * hh, a);
                tmem_wait_ld();
                if constexpr (kDecay) {
                    // lambda^(lim - col) for col <= lim (lim - col = row - key in the block), from the
                    // highest column of this half down: one power, then a product per kept column
                    float f = decay_pow(l2, max(lim - (32 * hh + 31), 0));
#pragma unroll
                    for (int q = 15; q >= 0; --q) {
                        const int c1 = 32 * hh + 2 * q + 1, c0 = c1 - 1;
                        const float x1 = c1 <= lim ? __uint_as_float(a[2 * q + 1]) * f : 0.f;
                        f = c1 <= lim ? f * lam : f;
                        const float x0 = c0 <= lim ? __uint_as_float(a[2 * q]) * f : 0.f;
                        f = c0 <= lim ? f * lam : f;
                        ph[q] = pack_bf16x2(x0, x1);
                    }
                } else if constexpr (kRev) {
                    // keys at or after the query row (col >= lim) and inside the sequence (col < hi)
                    const int hi = c.rows - KC * c.j - 64 * hk;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int c0 = 32 * hh + 2 * q;
                        ph[q] = pack_bf16x2(c0 >= lim && c0 < hi ? __uint_as_float(a[2 * q]) : 0.f,
                                            c0 + 1 >= lim && c0 + 1 < hi ? __uint_as_float(a[2 * q + 1]) : 0.f);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int c0 = 32 * hh + 2 * q;
                        ph[q] = pack_bf16x2(c0 <= lim ? __uint_as_float(a[2 * q]) : 0.f,
                                            c0 + 1 <= lim ? __uint_as_float(a[2 * q + 1]) : 0.f);
                    }
                }
                tmem_st_x16(ts + 16 * hh, ph);
            }
            if constexpr (kDecay) {
                if (c.first_of_sub()) {
                    // lambda^(r+1) q_r over the other 32 columns: head dims 64 hk .. 64 hk + 63 of
                    // query row m (the A operand of the inter-block MMA, read from TMEM)
                    const uint32_t qc = c.q0 + c.r;
                    if (!warp_all(wait_bar(&bars->q_full[qc % NQ], (qc / NQ) & 1, ab))) { ok = false; break; }
                    const uint8_t* qrow = smem + OFF_Q + (qc % NQ) * Q_BYTES + hk * QH_BYTES + m * 128;
                    const __nv_bfloat162 w2 = __float2bfloat162_rn(decay_pow(l2, UM * c.r + m + 1));
                    uint32_t qk[32];
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        uint4 u = *reinterpret_cast<const uint4*>(qrow + ((g ^ (m & 7)) << 4));
                        __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                        for (int x = 0; x < 4; ++x) e[x] = __hmul2(e[x], w2);
                        qk[4 * g] = u.x; qk[4 * g + 1] = u.y; qk[4 * g + 2] = u.z; qk[4 * g + 3] = u.w;
                    }
                    tmem_st_x32(ts + 32, qk);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[sbuf]);
            if (m == 0 && hk == 0 && c.k == 0) LA_CTRACE(c.n, TR_P0);
            if (m == 0 && hk == 0 && c.last_of_block()) LA_CTRACE(c.n, TR_PL);
            c.next_item(p);
        }
    } else if (warp >= 12 && warp < 16) {
        // ================================================================ state copy-out
        const int quad = warp & 3;
        const int m = quad * 32 + lane;                  // TMEM lane: state row i
        const int wt = threadIdx.x - 384;                // 0..127
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        uint8_t* sb = smem + OFF_SB;
        uint32_t kvc = 0;                                // blocks whose state was added
        bool ok = true;
        Cursor c;
        c.init(p);
        while (ok && c.valid) {
            if constexpr (kDecay) {
                // KV_b (or S0) -> bf16 operand of the inter-block product, one 32-column half at a
                // time straight into the shared buffer, and lambda^rows KV_b back into the
                // accumulator for this block's keys
                if (c.b > 0) {
                    if (!warp_all(wait_bar(&bars->kv_ready, kvc & 1, ab))) { ok = false; break; }
                    ++kvc;
                    tc_fence_after();
                }
                if (!warp_all(wait_bar(&bars->sb_empty, (c.n & 1) ^ 1, ab))) { ok = false; break; }
                const bool has = c.b > 0 || p.init != nullptr;
                const float wn = decay_pow(log2f(__ldg(p.decay + c.h)), c.rows);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t a[32];
                    if (c.b > 0) {
                        tmem_ld_x32(tmem + lane_base + TM_KV + 32 * hh, a);
                        tmem_wait_ld();
                    } else if (p.init) {
                        const float4* s0 = reinterpret_cast<const float4*>(
                            p.init + (((int64_t)c.seq * p.H + c.h) * D + m) * D + DV * c.half + 32 * hh);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 x = __ldg(s0 + q);
                            a[4 * q] = __float_as_uint(x.x);
                            a[4 * q + 1] = __float_as_uint(x.y);
                            a[4 * q + 2] = __float_as_uint(x.z);
                            a[4 * q + 3] = __float_as_uint(x.w);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) a[q] = 0u;
                    }
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int gg = 4 * hh + g;                      // 16-byte chunk of row m
                        *reinterpret_cast<uint4*>(sb + (m >> 3) * 1024 + (m & 7) * 128 + ((gg ^ (m & 7)) << 4)) =
                            make_uint4(pack_bf16x2(__uint_as_float(a[8 * g]), __uint_as_float(a[8 * g + 1])),
                                       pack_bf16x2(__uint_as_float(a[8 * g + 2]), __uint_as_float(a[8 * g + 3])),
                                       pack_bf16x2(__uint_as_float(a[8 * g + 4]), __uint_as_float(a[8 * g + 5])),
                                       pack_bf16x2(__uint_as_float(a[8 * g + 6]), __uint_as_float(a[8 * g + 7])));
                    }
                    if (has) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) a[q] = __float_as_uint(__uint_as_float(a[q]) * wn);
                        tmem_st_x32(tmem + lane_base + TM_KV + 32 * hh, a);
                    }
                }
                if (has) tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->kv_read[c.n & 3]);            // the accumulator may take this block's keys
                fence_proxy_async_smem();
                if (!(c.w == p.suppress_item && c.b == 1)) mbar_arrive(&bars->sb_full);
            } else {
            // KV_b -> bf16 operand of the inter-block product (row m, 64 columns)
            uint32_t pk[32];
            // anti-causal: the block walked after a ragged first block (the sequence's last)
            // takes that block's state on CUDA cores instead of from its (skipped) MMAs
            const int nbk = (c.bk.len + (1 << p.log2B) - 1) >> p.log2B;
            const bool ragged_next = kRev && !c.bk.first && c.b == nbk - 2 && (c.bk.len & ((1 << p.log2B) - 1)) != 0;
            if (ragged_next || !c.bk.first) {
                if (ragged_next) {
                    rev_ragged_state(p, tmem + lane_base + TM_KV, m, c.bk.tok_s + ((nbk - 1) << p.log2B),
                                     c.bk.tok_s + c.bk.len, c.h, c.half);
                } else {
                    if (!warp_all(wait_bar(&bars->kv_ready, kvc & 1, ab))) { ok = false; break; }
                    ++kvc;
                    if (wt == 0) LA_CTRACE(c.n, TR_XR);
                    tc_fence_after();
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t a[32];
                    tmem_ld_x32(tmem + lane_base + TM_KV + 32 * hh, a);
                    tmem_wait_ld();
                    if (hh == 1) {
                        tc_fence_before();
                        mbar_arrive(&bars->kv_read[c.n & 3]);    // the accumulator may take this block's keys
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        pk[16 * hh + q] = pack_bf16x2(__uint_as_float(a[2 * q]), __uint_as_float(a[2 * q + 1]));
                }
            } else {
                // A work item's first block: KV_0 = S0 (zero without a carried-in state).
                // S0 also seeds the accumulator, which the state MMAs then add onto, so
                // later prefixes already include it.
                if (p.init) {
                    const float* s0 = p.init + (((int64_t)c.seq * p.H + c.h) * D + m) * D + DV * c.half;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint32_t a[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 v = __ldg(reinterpret_cast<const float4*>(s0 + 32 * hh) + q);
                            a[4 * q] = __float_as_uint(v.x);
                            a[4 * q + 1] = __float_as_uint(v.y);
                            a[4 * q + 2] = __float_as_uint(v.z);
                            a[4 * q + 3] = __float_as_uint(v.w);
                        }
                        tmem_st_x32(tmem + lane_base + TM_KV + 32 * hh, a);
#pragma unroll
                        for (int q = 0; q < 16; ++q)
                            pk[16 * hh + q] = pack_bf16x2(__uint_as_float(a[2 * q]), __uint_as_float(a[2 * q + 1]));
                    }
                    tmem_wait_st();
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) pk[q] = 0u;
                }
                tc_fence_before();
                mbar_arrive(&bars->kv_read[c.n & 3]);            // the accumulator may take this block's keys
            }
            if (!warp_all(wait_bar(&bars->sb_empty, (c.n & 1) ^ 1, ab))) { ok = false; break; }
#pragma unroll
            for (int g = 0; g < 8; ++g)
                *reinterpret_cast<uint4*>(sb + (m >> 3) * 1024 + (m & 7) * 128 + ((g ^ (m & 7)) << 4)) =
                    make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
            fence_proxy_async_smem();
            if (!(c.w == p.suppress_item && c.b == 1)) mbar_arrive(&bars->sb_full);
            }
            if (wt == 0) LA_CTRACE(c.n, TR_SB);
            if (kStateOut && !c.add_state) {
                // the work item's last block: its state MMAs complete the final state
                if (!warp_all(wait_bar(&bars->kv_ready, kvc & 1, ab))) { ok = false; break; }
                ++kvc;
                tc_fence_after();
                // with no carried-in state and fewer than 16 tokens no MMA ever ran
                write_final_state<kDecay>(p, tmem + lane_base + TM_KV, m, p.init == nullptr && c.bk.len < 16,
                                          c.tok0 + (c.rows & ~15), c.tok0 + c.rows, c.seq, c.h, c.half);
            }
            c.next_block(p);
        }
    } else if (warp >= 16) {
        // ================================================================ O epilogue
        // (decay instance: also the weighted V copy of every chunk, one block ahead)
        const int quad = warp & 3;
        const int m = quad * 32 + lane;                  // TMEM lane: query row of the sub-unit
        const int wt = threadIdx.x - 512;                // 0..127
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        bool ok = true;
        Cursor c;
        c.init(p);
        Cursor cw;                                       // decay: the block whose V chunks are weighted next
        if constexpr (kDecay) {
            cw.init(p);
            ok = weight_block<kStateOut, SM>(cw, p, bars, smem, quad, lane, ab);
            if (cw.valid) cw.next_block(p);
        }
        while (ok && c.valid) {
            if constexpr (kDecay) {
                if (cw.valid) {
                    if (!weight_block<kStateOut, SM>(cw, p, bars, smem, quad, lane, ab)) break;
                    cw.next_block(p);
                }
            }
            // each sub-unit in the order the issuer finishes them
            for (int r = 0; ok && r < c.Rb; ++r) {
                const uint32_t slot = c.oslot(r);
                if (!warp_all(wait_bar(&bars->o_full[slot], c.ouse(r) & 1, ab))) { ok = false; break; }
                if (wt == 0) LA_CTRACE(c.n, r == 0 ? TR_E0 : TR_EL);
                tc_fence_after();
                uint32_t ov[32];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t a[32];
                    tmem_ld_x32(tmem + lane_base + TM_O + slot * 64 + 32 * hh, a);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        ov[16 * hh + q] = pack_bf16x2(__uint_as_float(a[2 * q]), __uint_as_float(a[2 * q + 1]));
                }
                tc_fence_before();
                mbar_arrive(&bars->o_empty[slot]);
                // row m: 64 bf16 = 128 contiguous bytes of token (tok0 + 128 r + m), head h
                if (m < c.rows - UM * r) {
                    __nv_bfloat16* orow = p.out + ((int64_t)(c.tok0 + UM * r + m) * p.H + c.h) * D + DV * c.half;
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        __stcs(reinterpret_cast<uint4*>(orow + 8 * g),
                               make_uint4(ov[4 * g], ov[4 * g + 1], ov[4 * g + 2], ov[4 * g + 3]));
                }
                if (wt == 0 && r == c.Rb - 1) LA_CTRACE(c.n, TR_ST);
            }
            c.next_block(p);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
    // every role has left its loop and every copy and MMA has completed (or the launch
    // aborted, in which case there is no decode work either)
    if constexpr (kStateOut) {
        if (p.ctrl->ok && !ab.raised()) singles_phase<kDecay>(p, smem, ab);
    }
    cluster_barrier();            // no remote store reaches a CTA that has ended
}

}  // namespace chain
}  // namespace la
