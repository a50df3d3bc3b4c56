// C ABI of the Lightning Attention library (declared in include/lightning_attention.h).
// Host side: argument validation, workspace layout, TMA tensor-map encoding and
// the launch sequence of each entry point. The whole library is this one
// translation unit (kernels come in through the .cuh files), so the per-device
// status word is a single __device__ symbol.
#include <cuda.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <stdint.h>
#include <string.h>

#include "lightning_attention.h"
#include "common.cuh"
#include "prep.cuh"
#include "simt.cuh"
#include "decode.cuh"
#include "fused.cuh"
#include "chain.cuh"
#include "state.cuh"
#include "lasp.cuh"
#include "backward.cuh"
#include "decay.cuh"

namespace {

using la::BlockEntry;
using la::Control;

constexpr uint64_t kWaitNs = 4000000000ull;   // bound on any single device-side wait (4 s)
constexpr int kStateBlock = 2048;             // tokens per partial state in la_state_from_prefill

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t esize(la_dtype t) { return t == LA_BF16 ? 2 : 4; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

bool supported_d(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }
bool supported_B(int B) { return B == 64 || B == 128 || B == 256; }
bool use_tensor_cores(la_dtype dt, int d, int B) { return dt == LA_BF16 && d == 128 && (B == 128 || B == 256); }

// Tensor-core prefill variants. The on-chip-state kernel gives one CTA to each
// (sequence, head, value-column half) and so needs enough of them to fill the
// GPU; below kChainMinItems work items the block-parallel look-back kernel
// (one CTA per SM over (block, head) tiles) is used instead.
enum class Path { simt, lookback, chain };
constexpr int64_t kChainMinItems = 64;
thread_local int t_force_path = 0;     // la_debug_set_path: 0 automatic, 1 on-chip state, 2 look-back

Path prefill_path(la_dtype dt, int d, int B, int nseq, int H) {
    if (!use_tensor_cores(dt, d, B)) return Path::simt;
    if (t_force_path == 1 && 2 * (int64_t)nseq * H < (int64_t(1) << 31)) return Path::chain;
    if (t_force_path == 2) return Path::lookback;
    const int64_t items = 2 * (int64_t)nseq * H;
    return items >= kChainMinItems && items < (int64_t(1) << 31) ? Path::chain : Path::lookback;
}

// ------------------------------------------------------------------ workspace layouts
struct Layout {
    int64_t max_blocks = 0, max_slots = 0;
    size_t off_seq_blk = 0, off_seq_slot = 0, off_table = 0, off_flags = 0, off_U = 0, off_prefix = 0,
           off_states = 0, off_seqs = 0, off_order = 0, total = 0;
    int nflag_arrays = 0;
};

// Control | seq_blk | seq_slot | block table, shared by every layout.
size_t layout_head(Layout& L, int64_t T, int nseq, int B) {
    L.max_blocks = (T + B - 1) / B + nseq;
    size_t off = sizeof(Control);
    L.off_seq_blk = off;  off = align_up(off + sizeof(int32_t) * (size_t)(nseq + 1), 256);
    L.off_seq_slot = off; off = align_up(off + sizeof(int32_t) * (size_t)(nseq + 1), 256);
    L.off_table = off;    off = align_up(off + sizeof(BlockEntry) * (size_t)L.max_blocks, 256);
    return off;
}

Layout prefill_layout(int64_t T, int nseq, int H, int d, int B, la_dtype dt) {
    Layout L;
    const Path path = prefill_path(dt, d, B, nseq, H);
    if (path == Path::chain) {
        // Control | sequence table | processing order
        size_t off = sizeof(Control);
        L.off_seqs = off;  off = align_up(off + sizeof(la::SeqEntry) * (size_t)nseq, 256);
        L.off_order = off; off = align_up(off + sizeof(int32_t) * (size_t)nseq, 256);
        L.total = off;
        return L;
    }
    size_t off = layout_head(L, T, nseq, B);
    const size_t dd = (size_t)d * d;
    if (path == Path::lookback) {
        // single pass: per-block flags (aggregate, inclusive, look-back done) and a
        // ring of kStateSlots published states per (sequence, head); a sequence with
        // n blocks uses min(n - 1, kStateSlots) slots.
        L.nflag_arrays = 3;
        L.off_flags = off;  off = align_up(off + sizeof(int32_t) * 3 * (size_t)L.max_blocks * H, 256);
        L.max_slots = std::min<int64_t>((int64_t)nseq * la::kStateSlots, (T + B - 1) / B);
        L.off_states = off; off = align_up(off + 2 * 4 * dd * (size_t)H * (size_t)L.max_slots, 256);
    } else {
        L.off_U = off;      off = align_up(off + 4 * dd * (size_t)H * (size_t)L.max_blocks, 256);
        L.off_prefix = off; off = align_up(off + 4 * dd * (size_t)H * (size_t)L.max_blocks, 256);
    }
    L.total = off;
    return L;
}

// The CUDA-core three-kernel prefill (block states, scan, prefill) whatever the
// dtype and shape: it also carries the decay variant.
Layout simt_layout(int64_t T, int nseq, int H, int d, int B) {
    Layout L;
    size_t off = layout_head(L, T, nseq, B);
    const size_t dd = (size_t)d * d;
    L.off_U = off;      off = align_up(off + 4 * dd * (size_t)H * (size_t)L.max_blocks, 256);
    L.off_prefix = off; off = align_up(off + 4 * dd * (size_t)H * (size_t)L.max_blocks, 256);
    L.total = off;
    return L;
}

// Block states of kStateBlock tokens and their scan (the CUDA-core state pass).
Layout simt_state_layout(int64_t T, int nseq, int H, int d);

Layout state_layout(int64_t T, int nseq, int H, int d, la_dtype dt) {
    Layout L;
    if (dt == LA_BF16 && d == 128) {
        // tensor-core path: Control | sequence table | order (unused here)
        size_t off = sizeof(Control);
        L.off_seqs = off;  off = align_up(off + sizeof(la::SeqEntry) * (size_t)nseq, 256);
        L.off_order = off; off = align_up(off + sizeof(int32_t) * (size_t)nseq, 256);
        L.total = off;
        return L;
    }
    return simt_state_layout(T, nseq, H, d);
}

Layout simt_state_layout(int64_t T, int nseq, int H, int d) {
    Layout L;
    size_t off = layout_head(L, T, nseq, kStateBlock);
    L.off_U = off; off = align_up(off + 4 * (size_t)d * d * (size_t)H * (size_t)L.max_blocks, 256);
    L.total = off;
    return L;
}

// ------------------------------------------------------------------ TMA tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [T][H][d] bf16 viewed as 3D {d, H, T}; box {64, 1, rows}, 128-byte swizzle.
bool map_tokens(CUtensorMap* m, const void* base, int64_t T, int H, int d, int rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

la_status cuda_check() { return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA; }

// Kernels launched by the library since the process started (la_launch_count).
std::atomic<uint64_t> g_launches{0};
inline void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Test hook (la_debug_set_fault): a tile that publishes nothing and a shorter wait limit.
thread_local long long t_suppress_tile = -1;
thread_local uint64_t t_wait_ns = 0;
// Debug trace buffer for the single-pass prefill (la_debug_set_trace).
thread_local uint64_t* t_trace = nullptr;
thread_local size_t t_trace_bytes = 0;

// One-shot per-thread timer around the main kernel of the next call (la_set_kernel_timer).
thread_local cudaEvent_t t_timer_start = nullptr, t_timer_stop = nullptr;

struct MainKernelTimer {
    cudaStream_t st;
    cudaEvent_t a, b;
    explicit MainKernelTimer(cudaStream_t s) : st(s), a(t_timer_start), b(t_timer_stop) {
        t_timer_start = t_timer_stop = nullptr;
        if (a) cudaEventRecord(a, st);
    }
    ~MainKernelTimer() {
        if (b) cudaEventRecord(b, st);
    }
};

// ------------------------------------------------------------------ launch helpers
la_status launch_block_table(const int32_t* cu, int nseq, int64_t T, int B, int H, const Layout& L, uint8_t* ws,
                             cudaStream_t st) {
    Control* ctrl = reinterpret_cast<Control*>(ws);
    int32_t* seq_blk = reinterpret_cast<int32_t*>(ws + L.off_seq_blk);
    int32_t* seq_slot = reinterpret_cast<int32_t*>(ws + L.off_seq_slot);
    BlockEntry* table = reinterpret_cast<BlockEntry*>(ws + L.off_table);
    int32_t* flags = L.nflag_arrays ? reinterpret_cast<int32_t*>(ws + L.off_flags) : nullptr;
    la::seq_blocks_kernel<<<1, 1024, 0, st>>>(cu, nseq, T, B, seq_blk, seq_slot, ctrl);
    note_launch();
    const int64_t nb = (L.max_blocks + 255) / 256;
    la::fill_block_table_kernel<<<(unsigned)nb, 256, 0, st>>>(cu, nseq, T, B, seq_blk, seq_slot, ctrl, table,
                                                              L.max_blocks, flags, L.nflag_arrays, H);
    note_launch();
    return cuda_check();
}

template <typename Tin, int D, bool kDecay>
la_status prefill_simt_main(const void* q, const void* k, const void* v, void* o, int H, int B,
                            const Layout& L, uint8_t* ws, const float* decay, cudaStream_t st) {
    const Control* ctrl = reinterpret_cast<const Control*>(ws);
    const BlockEntry* table = reinterpret_cast<const BlockEntry*>(ws + L.off_table);
    const float* prefix = reinterpret_cast<const float*>(ws + L.off_prefix);
    constexpr size_t smem = la::simt::prefill_simt_smem<D>();
    if (cudaFuncSetAttribute(la::simt::prefill_simt<Tin, D, kDecay>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return LA_ERR_CUDA;
    const int64_t grid = L.max_blocks * H * (B / 64);
    la::simt::prefill_simt<Tin, D, kDecay><<<(unsigned)grid, la::simt::THREADS, smem, st>>>(
        (const Tin*)q, (const Tin*)k, (const Tin*)v, (Tin*)o, prefix, table, ctrl, H, B, decay);
    note_launch();
    return cuda_check();
}

template <typename Tin, int D, bool kDecay>
la_status state_simt_launch(const void* k, const void* v, int H, const Layout& L, uint8_t* ws, const float* decay,
                            cudaStream_t st) {
    const Control* ctrl = reinterpret_cast<const Control*>(ws);
    const BlockEntry* table = reinterpret_cast<const BlockEntry*>(ws + L.off_table);
    float* U = reinterpret_cast<float*>(ws + L.off_U);
    la::simt::block_state_simt<Tin, D, kDecay><<<(unsigned)(L.max_blocks * H), la::simt::THREADS, 0, st>>>(
        (const Tin*)k, (const Tin*)v, table, ctrl, H, U, decay);
    note_launch();
    return cuda_check();
}

#define LA_DISPATCH_D(d, FN, ...)                          \
    switch (d) {                                           \
        case 16: return FN<16>(__VA_ARGS__);               \
        case 32: return FN<32>(__VA_ARGS__);               \
        case 48: return FN<48>(__VA_ARGS__);               \
        case 64: return FN<64>(__VA_ARGS__);               \
        case 80: return FN<80>(__VA_ARGS__);               \
        case 96: return FN<96>(__VA_ARGS__);               \
        case 112: return FN<112>(__VA_ARGS__);             \
        case 128: return FN<128>(__VA_ARGS__);             \
        default: return LA_ERR_UNSUPPORTED;                \
    }

// The instances with a decay rate per head (decay.cuh) are chosen by decay != nullptr.
template <int D>
la_status simt_states(la_dtype dt, const void* k, const void* v, int H, const Layout& L, uint8_t* ws,
                      const float* decay, cudaStream_t st) {
    if (decay)
        return dt == LA_BF16 ? state_simt_launch<__nv_bfloat16, D, true>(k, v, H, L, ws, decay, st)
                             : state_simt_launch<float, D, true>(k, v, H, L, ws, decay, st);
    return dt == LA_BF16 ? state_simt_launch<__nv_bfloat16, D, false>(k, v, H, L, ws, nullptr, st)
                         : state_simt_launch<float, D, false>(k, v, H, L, ws, nullptr, st);
}

template <int D>
la_status simt_prefill(la_dtype dt, const void* q, const void* k, const void* v, void* o, int H, int B,
                       const Layout& L, uint8_t* ws, const float* decay, cudaStream_t st) {
    if (decay)
        return dt == LA_BF16 ? prefill_simt_main<__nv_bfloat16, D, true>(q, k, v, o, H, B, L, ws, decay, st)
                             : prefill_simt_main<float, D, true>(q, k, v, o, H, B, L, ws, decay, st);
    return dt == LA_BF16 ? prefill_simt_main<__nv_bfloat16, D, false>(q, k, v, o, H, B, L, ws, nullptr, st)
                         : prefill_simt_main<float, D, false>(q, k, v, o, H, B, L, ws, nullptr, st);
}

template <typename Tin, int D, bool kDecay>
void decode_instance(const void* q, const void* k, const void* v, float* state, void* o, int64_t pairs,
                     const float* decay, int H, cudaStream_t st) {
    constexpr int nt = (D / 4) * la::decode_row_groups(D);
    la::decode_step_kernel<Tin, D, kDecay><<<(unsigned)pairs, nt, 0, st>>>(
        (const Tin*)q, (const Tin*)k, (const Tin*)v, state, (Tin*)o, decay, H);
}

template <int D>
la_status decode_launch(la_dtype dt, const void* q, const void* k, const void* v, float* state, void* o,
                        int64_t pairs, const float* decay, int H, cudaStream_t st) {
    if (dt == LA_BF16)
        decay ? decode_instance<__nv_bfloat16, D, true>(q, k, v, state, o, pairs, decay, H, st)
              : decode_instance<__nv_bfloat16, D, false>(q, k, v, state, o, pairs, nullptr, H, st);
    else
        decay ? decode_instance<float, D, true>(q, k, v, state, o, pairs, decay, H, st)
              : decode_instance<float, D, false>(q, k, v, state, o, pairs, nullptr, H, st);
    note_launch();
    return cuda_check();
}

la_status simt_states_d(int d, la_dtype dt, const void* k, const void* v, int H, const Layout& L, uint8_t* ws,
                        const float* decay, cudaStream_t st) {
    LA_DISPATCH_D(d, simt_states, dt, k, v, H, L, ws, decay, st);
}
la_status simt_prefill_d(int d, la_dtype dt, const void* q, const void* k, const void* v, void* o, int H, int B,
                         const Layout& L, uint8_t* ws, const float* decay, cudaStream_t st) {
    LA_DISPATCH_D(d, simt_prefill, dt, q, k, v, o, H, B, L, ws, decay, st);
}
la_status decode_d(int d, la_dtype dt, const void* q, const void* k, const void* v, float* state, void* o,
                   int64_t pairs, const float* decay, int H, cudaStream_t st) {
    LA_DISPATCH_D(d, decode_launch, dt, q, k, v, state, o, pairs, decay, H, st);
}

// Common argument checks of the token-major entry points.
la_status check_tokens(int64_t T, int nseq, int H, int d, la_dtype dt, const int32_t* cu) {
    if (T < 0 || H < 1 || nseq < 1) return LA_ERR_INVALID_ARGUMENT;
    if (cu == nullptr && nseq != 1) return LA_ERR_INVALID_ARGUMENT;
    if (dt != LA_BF16 && dt != LA_FP32) return LA_ERR_UNSUPPORTED;
    if (!supported_d(d)) return LA_ERR_UNSUPPORTED;
    if (T >= (int64_t(1) << 31)) return LA_ERR_UNSUPPORTED;    // int32 cu_seqlens
    if (cu && !aligned(cu, 4)) return LA_ERR_MISALIGNED;
    return LA_OK;
}

// The on-chip-state prefill (bf16, d = 128): sequence table, then the kernel;
// with state_out, the instance that also writes the final states.
// Rates of the decay variant (nullptr: none) are checked on the device first.
la_status launch_decay_check(const float* decay, int heads, uint8_t* ws, cudaStream_t st) {
    la::decay_check_kernel<<<1, 256, 0, st>>>(decay, heads, reinterpret_cast<Control*>(ws));
    note_launch();
    return cuda_check();
}

// 2-CTA clusters of the on-chip-state kernel that fit on the device at once (cached per
// device): the grid stays within them, so no cluster waits for another to finish.
int chain_max_clusters() {
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int n = 0;
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(la::chain::NTHREADS, 1, 1);
        cfg.dynamicSmemBytes = la::chain::Smem<true>::BYTES;   // the larger of the instances
        cfg.gridDim = dim3(2 * 74, 1, 1);
        if (cudaFuncSetAttribute(la::chain::prefill_chain_kernel<true, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cfg.dynamicSmemBytes) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, la::chain::prefill_chain_kernel<true, true>, &cfg) != cudaSuccess ||
            n <= 0) {
            cudaGetLastError();
            n = num_sms() / 2;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

// rev: the anti-causal instance (O_t = q_t S0 + sum_{s >= t} (q_t . k_s) v_s; no state output,
// no decay), which the backward pass uses for dk and dv.
la_status launch_chain(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens, int num_seqs,
                       int64_t total_tokens, int heads, int d, int B, const float* init_state, float* state_out,
                       uint8_t* ws, const Layout& L, cudaStream_t st, const float* decay = nullptr, bool rev = false) {
    la_status s;
    const Control* ctrl = reinterpret_cast<const Control*>(ws);
    la::SeqEntry* seqs = reinterpret_cast<la::SeqEntry*>(ws + L.off_seqs);
    int32_t* order = reinterpret_cast<int32_t*>(ws + L.off_order);
    la::seq_table_kernel<<<1, 1024, 0, st>>>(cu_seqlens, num_seqs, total_tokens, seqs, order,
                                             reinterpret_cast<Control*>(ws));
    note_launch();
    if ((s = cuda_check()) != LA_OK) return s;
    if (decay && (s = launch_decay_check(decay, heads, ws, st)) != LA_OK) return s;
    if (state_out && init_state != state_out) {
        const int64_t per_seq4 = (int64_t)heads * d * d / 4;
        const int sms = num_sms();
        if (sms <= 0) return LA_ERR_CUDA;
        la::empty_states_kernel<<<(unsigned)std::min<int64_t>(num_seqs, (int64_t)sms * 8), 256, 0, st>>>(
            seqs, num_seqs, per_seq4, reinterpret_cast<const float4*>(init_state), reinterpret_cast<float4*>(state_out),
            ctrl);
        note_launch();
        if ((s = cuda_check()) != LA_OK) return s;
    }
    CUtensorMap tq, tk, tv;
    if (!map_tokens(&tq, q, total_tokens, heads, d, la::chain::UM) ||
        !map_tokens(&tk, k, total_tokens, heads, d, la::chain::KC) ||
        !map_tokens(&tv, v, total_tokens, heads, d, la::chain::KC))
        return LA_ERR_CUDA;
    la::chain::Params prm;
    prm.out = static_cast<__nv_bfloat16*>(o);
    prm.seqs = seqs;
    prm.order = order;
    prm.ctrl = ctrl;
    prm.init = init_state;
    prm.state_out = state_out;
    prm.k = static_cast<const __nv_bfloat16*>(k);
    prm.v = static_cast<const __nv_bfloat16*>(v);
    prm.q = static_cast<const __nv_bfloat16*>(q);
    prm.H = heads;
    prm.B = B;
    prm.log2B = B == 256 ? 8 : 7;
    prm.nseq = num_seqs;
    prm.wait_ns = t_wait_ns ? t_wait_ns : kWaitNs;
    prm.suppress_item = t_suppress_tile;
    prm.decay = decay;
    // items come in (value half 0, value half 1) pairs: an even grid of 2-CTA clusters
    const int64_t items = 2 * (int64_t)num_seqs * heads;
    const int clusters = chain_max_clusters();
    if (clusters <= 0) return LA_ERR_CUDA;
    const unsigned grid = (unsigned)(items < 2 * (int64_t)clusters ? items : 2 * (int64_t)clusters);
    const size_t per_block = (size_t)grid * la::chain::kTraceEvents * sizeof(uint64_t);
    prm.trace = (t_trace && t_trace_bytes >= per_block) ? t_trace : nullptr;
    prm.trace_blocks = prm.trace ? (int)std::min<size_t>(t_trace_bytes / per_block, 1 << 30) : 0;
    if (rev && (decay || state_out)) return LA_ERR_UNSUPPORTED;
    auto kernel = rev ? la::chain::prefill_chain_kernel<false, false, true>
                : decay ? (state_out ? la::chain::prefill_chain_kernel<true, true>
                                     : la::chain::prefill_chain_kernel<false, true>)
                        : (state_out ? la::chain::prefill_chain_kernel<true, false>
                                     : la::chain::prefill_chain_kernel<false, false>);
    const uint32_t smem = decay ? la::chain::Smem<true>::BYTES : la::chain::Smem<false>::BYTES;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return LA_ERR_CUDA;
    MainKernelTimer timer(st);
    kernel<<<grid, la::chain::NTHREADS, smem, st>>>(tq, tk, tv, prm);
    note_launch();
    return cuda_check();
}

// Workspace of la_prefill_backward: four reversed inputs, one reversed output,
// S0^T, and the workspaces of the prefill and of the state pass.
struct BackwardLayout {
    size_t tensor = 0, off_rk = 0, off_rq = 0, off_rdo = 0, off_rv = 0, off_rout = 0, off_s0t = 0, off_pws = 0,
           pws = 0, off_sws = 0, sws = 0, total = 0;
};
Layout simt_layout(int64_t T, int nseq, int H, int d, int B);
// dk and dv by the anti-causal instance of the on-chip-state kernel (no sequence
// reversals) wherever the forward prefill takes that kernel, without decay.
bool backward_in_place_order(la_dtype dt, int d, int B, int nseq, int H, bool decay) {
    return !decay && prefill_path(dt, d, B, nseq, H) == Path::chain;
}
BackwardLayout backward_layout(int64_t T, int nseq, int H, int d, int B, la_dtype dt, bool decay = false) {
    BackwardLayout L;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    // the reversed copies are needed only when dk and dv come from prefills of reversed sequences
    L.tensor = backward_in_place_order(dt, d, B, nseq, H, decay) ? 0 : (size_t)T * H * d * esize(dt);
    size_t off = 0;
    L.off_rk = off; off = up(off + L.tensor);
    L.off_rq = off; off = up(off + L.tensor);
    L.off_rdo = off; off = up(off + L.tensor);
    L.off_rv = off; off = up(off + L.tensor);
    L.off_rout = off; off = up(off + L.tensor);
    L.off_s0t = off; off = up(off + (size_t)nseq * H * d * d * 4);
    if (decay)   // the workspaces of la_prefill_decay and la_state_decay
        L.pws = T > 0 && prefill_path(dt, d, B, nseq, H) == Path::chain ? prefill_layout(T, nseq, H, d, B, dt).total
                                                                        : simt_layout(T, nseq, H, d, B).total;
    else
        L.pws = prefill_layout(T, nseq, H, d, B, dt).total;
    L.off_pws = off; off = up(off + L.pws);
    L.sws = decay ? simt_state_layout(T, nseq, H, d).total : state_layout(T, nseq, H, d, dt).total;
    L.off_sws = off; off = up(off + L.sws);
    L.total = off;
    return L;
}

la_status launch_reverse(const void* in, void* out, const int32_t* cu, int nseq, int64_t T, int H, int d, la_dtype dt,
                         cudaStream_t st) {
    const int64_t row16 = (int64_t)H * d * esize(dt) / 16;
    const int sms = num_sms();
    if (sms <= 0) return LA_ERR_CUDA;
    const dim3 grid((unsigned)(2 * sms), (unsigned)std::min(nseq, 65535));
    la::reverse_tokens_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(in), static_cast<uint4*>(out), cu, nseq,
                                                    T, row16);
    note_launch();
    return cuda_check();
}

// The host checks of la_prefill's arguments (workspace excluded).
la_status check_prefill(const void* q, const void* k, const void* v, const void* o, const int32_t* cu_seqlens,
                        int num_seqs, int64_t total_tokens, int heads, int d, int B, la_dtype dtype,
                        const float* init_state) {
    la_status s = check_tokens(total_tokens, num_seqs, heads, d, dtype, cu_seqlens);
    if (s != LA_OK) return s;
    if (!supported_B(B)) return LA_ERR_UNSUPPORTED;
    const size_t tensor_bytes = (size_t)total_tokens * heads * d * esize(dtype);
    if (total_tokens > 0 && (!q || !k || !v || !o)) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return LA_ERR_MISALIGNED;
    if (init_state && !aligned(init_state, 16)) return LA_ERR_MISALIGNED;
    if (overlaps(o, tensor_bytes, q, tensor_bytes) || overlaps(o, tensor_bytes, k, tensor_bytes) ||
        overlaps(o, tensor_bytes, v, tensor_bytes))
        return LA_ERR_INVALID_ARGUMENT;
    return LA_OK;
}

}  // namespace

extern "C" {

size_t la_prefill_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B, la_dtype dtype) {
    if (total_tokens < 0 || num_seqs < 1 || heads < 1 || !supported_d(d) || !supported_B(B) ||
        (dtype != LA_BF16 && dtype != LA_FP32))
        return 0;
    return prefill_layout(total_tokens, num_seqs, heads, d, B, dtype).total;
}

size_t la_state_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, la_dtype dtype) {
    if (total_tokens < 0 || num_seqs < 1 || heads < 1 || !supported_d(d) || (dtype != LA_BF16 && dtype != LA_FP32))
        return 0;
    return state_layout(total_tokens, num_seqs, heads, d, dtype).total;
}

la_status la_prefill(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                     int num_seqs, int64_t total_tokens, int heads, int d, int B, la_dtype dtype,
                     const float* init_state, void* workspace, size_t workspace_bytes, void* stream) {
    la_status s = check_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state);
    if (s != LA_OK) return s;
    const size_t tensor_bytes = (size_t)total_tokens * heads * d * esize(dtype);
    if (total_tokens == 0) return LA_OK;
    const Layout L = prefill_layout(total_tokens, num_seqs, heads, d, B, dtype);
    if (!workspace) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(workspace, 256)) return LA_ERR_MISALIGNED;
    if (workspace_bytes < L.total) return LA_ERR_WORKSPACE_TOO_SMALL;
    if (overlaps(workspace, L.total, o, tensor_bytes)) return LA_ERR_INVALID_ARGUMENT;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const Control* ctrl = reinterpret_cast<const Control*>(ws);
    const Path path = prefill_path(dtype, d, B, num_seqs, heads);

    if (path == Path::chain)
        return launch_chain(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, init_state, nullptr, ws, L, st);

    const int32_t* seq_blk = reinterpret_cast<const int32_t*>(ws + L.off_seq_blk);
    const BlockEntry* table = reinterpret_cast<const BlockEntry*>(ws + L.off_table);
    float* U = reinterpret_cast<float*>(ws + L.off_U);
    const int dd = d * d;

    if ((s = launch_block_table(cu_seqlens, num_seqs, total_tokens, B, heads, L, ws, st)) != LA_OK) return s;

    if (path == Path::lookback) {
        CUtensorMap tq, tk, tv, to;
        if (!map_tokens(&tq, q, total_tokens, heads, d, 128) || !map_tokens(&tk, k, total_tokens, heads, d, 64) ||
            !map_tokens(&tv, v, total_tokens, heads, d, 64) || !map_tokens(&to, o, total_tokens, heads, d, 128))
            return LA_ERR_CUDA;
        la::fused::Params prm;
        prm.out = static_cast<__nv_bfloat16*>(o);
        prm.table = table;
        prm.ctrl = ctrl;
        int32_t* flags = reinterpret_cast<int32_t*>(ws + L.off_flags);
        prm.agg_flag = flags;
        prm.incl_flag = flags + L.max_blocks * heads;
        prm.lb_done = flags + 2 * L.max_blocks * heads;
        prm.states = reinterpret_cast<float*>(ws + L.off_states);
        prm.init = init_state;
        prm.H = heads;
        prm.R = B / 128;
        prm.wait_ns = t_wait_ns ? t_wait_ns : kWaitNs;
        prm.suppress_tile = t_suppress_tile;
        const size_t trace_need = (size_t)L.max_blocks * heads * la::fused::kTraceEvents * sizeof(uint64_t);
        prm.trace = (t_trace && t_trace_bytes >= trace_need) ? t_trace : nullptr;
        prm.grace_ns = 1500;
        if (cudaFuncSetAttribute(la::fused::prefill_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)la::fused::SMEM_BYTES) != cudaSuccess)
            return LA_ERR_CUDA;
        const int64_t tiles = L.max_blocks * heads;
        const int sms = num_sms();
        if (sms <= 0) return LA_ERR_CUDA;
        const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
        MainKernelTimer timer(st);
        la::fused::prefill_fused_kernel<<<grid, la::fused::NTHREADS, la::fused::SMEM_BYTES, st>>>(tq, tk, tv, to,
                                                                                                   prm);
        note_launch();
        return cuda_check();
    }

    // CUDA-core path
    if ((s = simt_states_d(d, dtype, k, v, heads, L, ws, nullptr, st)) != LA_OK) return s;
    dim3 sg((dd + 1023) / 1024, num_seqs * heads);
    la::chain_scan_kernel<float><<<sg, 256, 0, st>>>(U, reinterpret_cast<float*>(ws + L.off_prefix), init_state,
                                                     nullptr, seq_blk, ctrl, num_seqs, heads, dd, true, table,
                                                     nullptr);
    note_launch();
    if ((s = cuda_check()) != LA_OK) return s;
    MainKernelTimer timer(st);
    return simt_prefill_d(d, dtype, q, k, v, o, heads, B, L, ws, nullptr, st);
}

la_status la_state_from_prefill(const void* k, const void* v, const int32_t* cu_seqlens, int num_seqs,
                                int64_t total_tokens, int heads, int d, la_dtype dtype, const float* init_state,
                                float* state_out, void* workspace, size_t workspace_bytes, void* stream) {
    la_status s = check_tokens(total_tokens, num_seqs, heads, d, dtype, cu_seqlens);
    if (s != LA_OK) return s;
    if (!state_out || (total_tokens > 0 && (!k || !v))) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(state_out, 16)) return LA_ERR_MISALIGNED;
    if (init_state && !aligned(init_state, 16)) return LA_ERR_MISALIGNED;
    const size_t state_bytes = (size_t)num_seqs * heads * d * d * 4;
    if (init_state && init_state != state_out && overlaps(init_state, state_bytes, state_out, state_bytes))
        return LA_ERR_INVALID_ARGUMENT;
    const Layout L = state_layout(total_tokens, num_seqs, heads, d, dtype);
    if (!workspace) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(workspace, 256)) return LA_ERR_MISALIGNED;
    if (workspace_bytes < L.total) return LA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (dtype == LA_BF16 && d == 128) {
        // tensor cores: one CTA per (sequence, head, value-column half)
        la::SeqEntry* seqs = reinterpret_cast<la::SeqEntry*>(ws + L.off_seqs);
        la::seq_table_kernel<<<1, 1024, 0, st>>>(cu_seqlens, num_seqs, total_tokens, seqs,
                                                 reinterpret_cast<int32_t*>(ws + L.off_order),
                                                 reinterpret_cast<Control*>(ws));
        note_launch();
        if ((s = cuda_check()) != LA_OK) return s;
        CUtensorMap tk, tv;
        const int64_t rows = total_tokens > 0 ? total_tokens : 1;
        if (!map_tokens(&tk, k ? k : state_out, rows, heads, d, la::state::KC) ||
            !map_tokens(&tv, v ? v : state_out, rows, heads, d, la::state::KC))
            return LA_ERR_CUDA;
        la::state::Params prm;
        prm.out = state_out;
        prm.init = init_state;
        prm.seqs = seqs;
        prm.ctrl = reinterpret_cast<const Control*>(ws);
        prm.H = heads;
        prm.nseq = num_seqs;
        prm.wait_ns = t_wait_ns ? t_wait_ns : kWaitNs;
        if (cudaFuncSetAttribute(la::state::state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)la::state::SMEM_BYTES) != cudaSuccess)
            return LA_ERR_CUDA;
        const int64_t items = 2 * (int64_t)num_seqs * heads;
        const int sms = num_sms();
        if (sms <= 0) return LA_ERR_CUDA;
        const unsigned grid = (unsigned)(items < sms ? items : sms);
        la::state::state_kernel<<<grid, la::state::NTHREADS, la::state::SMEM_BYTES, st>>>(tk, tv, prm);
        note_launch();
        return cuda_check();
    }
    if ((s = launch_block_table(cu_seqlens, num_seqs, total_tokens, kStateBlock, heads, L, ws, st)) != LA_OK) return s;
    if (total_tokens > 0 && (s = simt_states_d(d, dtype, k, v, heads, L, ws, nullptr, st)) != LA_OK) return s;
    const int dd = d * d;
    dim3 sg((dd + 1023) / 1024, num_seqs * heads);
    la::chain_scan_kernel<float><<<sg, 256, 0, st>>>(
        reinterpret_cast<const float*>(ws + L.off_U), static_cast<float*>(nullptr), init_state, state_out,
        reinterpret_cast<const int32_t*>(ws + L.off_seq_blk), reinterpret_cast<const Control*>(ws), num_seqs,
        heads, dd, false, reinterpret_cast<const BlockEntry*>(ws + L.off_table), nullptr);
    note_launch();
    return cuda_check();
}

la_status la_decode_step(const void* q, const void* k, const void* v, float* state, void* o, int batch, int heads,
                         int d, la_dtype dtype, void* stream) {
    if (batch < 0 || heads < 1) return LA_ERR_INVALID_ARGUMENT;
    if (dtype != LA_BF16 && dtype != LA_FP32) return LA_ERR_UNSUPPORTED;
    if (!supported_d(d)) return LA_ERR_UNSUPPORTED;
    if (batch == 0) return LA_OK;
    if (!q || !k || !v || !state || !o) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(state, 16))
        return LA_ERR_MISALIGNED;
    const int64_t pairs = (int64_t)batch * heads;
    const size_t vec = (size_t)pairs * d * esize(dtype);
    const size_t sbytes = (size_t)pairs * d * d * 4;
    if (overlaps(o, vec, q, vec) || overlaps(o, vec, k, vec) || overlaps(o, vec, v, vec) ||
        overlaps(o, vec, state, sbytes) || overlaps(state, sbytes, q, vec) || overlaps(state, sbytes, k, vec) ||
        overlaps(state, sbytes, v, vec))
        return LA_ERR_INVALID_ARGUMENT;
    if (pairs >= (int64_t(1) << 31)) return LA_ERR_UNSUPPORTED;
    MainKernelTimer timer(reinterpret_cast<cudaStream_t>(stream));
    return decode_d(d, dtype, q, k, v, state, o, pairs, nullptr, heads, reinterpret_cast<cudaStream_t>(stream));
}

la_status la_state_exclusive_prefix_decay(const float* gathered, const int32_t* seg_lens, int world, int rank,
                                          int num_seqs, int heads, int d, const float* decay, const float* init,
                                          float* out, void* stream) {
    if (world < 1 || rank < 0 || rank > world || num_seqs < 0 || heads < 1) return LA_ERR_INVALID_ARGUMENT;
    if (!supported_d(d)) return LA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return LA_OK;
    if (!gathered || !out || !decay || (rank > 0 && !seg_lens)) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(gathered, 16) || !aligned(out, 16) || (init && !aligned(init, 16)) || !aligned(decay, 4) ||
        (seg_lens && !aligned(seg_lens, 4)))
        return LA_ERR_MISALIGNED;
    const int64_t per_state = (int64_t)d * d;
    const int64_t per_rank = (int64_t)num_seqs * heads * per_state;
    const size_t bytes = (size_t)per_rank * 4;
    if (overlaps(out, bytes, gathered, bytes * (size_t)world)) return LA_ERR_INVALID_ARGUMENT;
    if (init && init != out && overlaps(out, bytes, init, bytes)) return LA_ERR_INVALID_ARGUMENT;
    if (overlaps(out, bytes, decay, (size_t)heads * 4) ||
        (seg_lens && overlaps(out, bytes, seg_lens, (size_t)world * num_seqs * 4)))
        return LA_ERR_INVALID_ARGUMENT;
    const int sms = num_sms();
    if (sms <= 0) return LA_ERR_CUDA;
    const int64_t per_rank4 = per_rank / 4;
    const int64_t want = (per_rank4 + 255) / 256;
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)sms * 8);
    la::state_prefix_decay_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float4*>(gathered), seg_lens, rank, num_seqs, heads, per_state / 4, per_rank4, decay,
        reinterpret_cast<const float4*>(init), reinterpret_cast<float4*>(out));
    note_launch();
    return cuda_check();
}

la_status la_state_exclusive_prefix(const float* gathered, int world, int rank, int64_t n, int d, const float* init,
                                    float* out, void* stream) {
    if (world < 1 || rank < 0 || rank > world || n < 0) return LA_ERR_INVALID_ARGUMENT;
    if (!supported_d(d)) return LA_ERR_UNSUPPORTED;
    if (n == 0) return LA_OK;
    if (!gathered || !out) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(gathered, 16) || !aligned(out, 16) || (init && !aligned(init, 16))) return LA_ERR_MISALIGNED;
    const int64_t per_rank = n * d * d;                 // floats of one rank's states
    const size_t bytes = (size_t)per_rank * 4;
    if (overlaps(out, bytes, gathered, bytes * (size_t)world)) return LA_ERR_INVALID_ARGUMENT;
    if (init && init != out && overlaps(out, bytes, init, bytes)) return LA_ERR_INVALID_ARGUMENT;
    const int sms = num_sms();
    if (sms <= 0) return LA_ERR_CUDA;
    const int64_t per_rank4 = per_rank / 4;             // d*d is a multiple of 4 for every supported d
    const int64_t want = (per_rank4 + 255) / 256;
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)sms * 8);
    la::state_prefix_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float4*>(gathered), rank, per_rank4, reinterpret_cast<const float4*>(init),
        reinterpret_cast<float4*>(out));
    note_launch();
    return cuda_check();
}

size_t la_prefill_with_state_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                            la_dtype dtype) {
    const size_t a = la_prefill_workspace_size(total_tokens, num_seqs, heads, d, B, dtype);
    const size_t b = la_state_workspace_size(total_tokens, num_seqs, heads, d, dtype);
    return (a == 0 || b == 0) ? 0 : std::max(a, b);
}

la_status la_prefill_with_state(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                                int num_seqs, int64_t total_tokens, int heads, int d, int B, la_dtype dtype,
                                const float* init_state, float* state_out, void* workspace, size_t workspace_bytes,
                                void* stream) {
    la_status s = check_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state);
    if (s != LA_OK) return s;
    if (!state_out) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(state_out, 16)) return LA_ERR_MISALIGNED;
    const size_t tb = (size_t)total_tokens * heads * d * esize(dtype);
    const size_t sb = (size_t)num_seqs * heads * d * d * 4;
    // state_out may be init_state itself (the state is read before it is written, per slice)
    if (init_state && init_state != state_out && overlaps(state_out, sb, init_state, sb)) return LA_ERR_INVALID_ARGUMENT;
    if (overlaps(state_out, sb, o, tb) || overlaps(state_out, sb, q, tb) || overlaps(state_out, sb, k, tb) ||
        overlaps(state_out, sb, v, tb))
        return LA_ERR_INVALID_ARGUMENT;
    if (workspace && overlaps(workspace, workspace_bytes, state_out, sb)) return LA_ERR_INVALID_ARGUMENT;
    if (total_tokens > 0 && prefill_path(dtype, d, B, num_seqs, heads) == Path::chain) {
        // one pass: the prefill kernel's state-output instance
        const Layout L = prefill_layout(total_tokens, num_seqs, heads, d, B, dtype);
        if (!workspace) return LA_ERR_INVALID_ARGUMENT;
        if (!aligned(workspace, 256)) return LA_ERR_MISALIGNED;
        if (workspace_bytes < L.total) return LA_ERR_WORKSPACE_TOO_SMALL;
        if (overlaps(workspace, L.total, o, tb)) return LA_ERR_INVALID_ARGUMENT;
        return launch_chain(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, init_state, state_out,
                            static_cast<uint8_t*>(workspace), L, reinterpret_cast<cudaStream_t>(stream));
    }
    // other paths: the prefill, then the state pass (stream order keeps init_state valid until both read it)
    if (init_state == state_out && init_state) {
        // the state pass accumulates in place; the prefill reads S0 first
        if ((s = la_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state, workspace,
                            workspace_bytes, stream)) != LA_OK)
            return s;
        return la_state_from_prefill(k, v, cu_seqlens, num_seqs, total_tokens, heads, d, dtype, state_out, state_out,
                                     workspace, workspace_bytes, stream);
    }
    if ((s = la_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state, workspace,
                        workspace_bytes, stream)) != LA_OK)
        return s;
    return la_state_from_prefill(k, v, cu_seqlens, num_seqs, total_tokens, heads, d, dtype, init_state, state_out,
                                 workspace, workspace_bytes, stream);
}

size_t la_prefill_backward_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                          la_dtype dtype) {
    if (la_prefill_workspace_size(total_tokens, num_seqs, heads, d, B, dtype) == 0) return 0;
    return backward_layout(total_tokens, num_seqs, heads, d, B, dtype).total;
}

static la_status prefill_backward_impl(const void* q, const void* k, const void* v, const void* dout,
                                const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, int heads, int d,
                                int B, la_dtype dtype, const float* init_state, const float* decay, void* dq,
                                void* dk, void* dv, float* dinit_state, void* workspace, size_t workspace_bytes,
                                void* stream);

la_status la_prefill_backward(const void* q, const void* k, const void* v, const void* dout,
                              const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, int heads, int d, int B,
                              la_dtype dtype, const float* init_state, void* dq, void* dk, void* dv,
                              float* dinit_state, void* workspace, size_t workspace_bytes, void* stream) {
    return prefill_backward_impl(q, k, v, dout, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state,
                                 nullptr, dq, dk, dv, dinit_state, workspace, workspace_bytes, stream);
}

size_t la_prefill_backward_decay_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B,
                                                la_dtype dtype) {
    if (la_prefill_decay_workspace_size(total_tokens, num_seqs, heads, d, B, dtype) == 0) return 0;
    return backward_layout(total_tokens, num_seqs, heads, d, B, dtype, true).total;
}

la_status la_prefill_backward_decay(const void* q, const void* k, const void* v, const void* dout,
                                    const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, int heads, int d,
                                    int B, la_dtype dtype, const float* init_state, const float* decay, void* dq,
                                    void* dk, void* dv, float* dinit_state, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    if (!decay) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(decay, 4)) return LA_ERR_MISALIGNED;
    return prefill_backward_impl(q, k, v, dout, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state,
                                 decay, dq, dk, dv, dinit_state, workspace, workspace_bytes, stream);
}

}  // extern "C"

// The backward pass without (decay = nullptr) or with a decay rate per head.
static la_status prefill_backward_impl(const void* q, const void* k, const void* v, const void* dout,
                                const int32_t* cu_seqlens, int num_seqs, int64_t total_tokens, int heads, int d,
                                int B, la_dtype dtype, const float* init_state, const float* decay, void* dq,
                                void* dk, void* dv, float* dinit_state, void* workspace, size_t workspace_bytes,
                                void* stream) {
    la_status s = check_tokens(total_tokens, num_seqs, heads, d, dtype, cu_seqlens);
    if (s != LA_OK) return s;
    if (!supported_B(B)) return LA_ERR_UNSUPPORTED;
    const int64_t T = total_tokens;
    const size_t tb = (size_t)T * heads * d * esize(dtype);
    const size_t sb = (size_t)num_seqs * heads * d * d * 4;
    if (T > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv)) return LA_ERR_INVALID_ARGUMENT;
    for (const void* p : {q, k, v, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
        if (!aligned(p, 16)) return LA_ERR_MISALIGNED;
    if ((init_state && !aligned(init_state, 16)) || (dinit_state && !aligned(dinit_state, 16))) return LA_ERR_MISALIGNED;
    const void* outs[3] = {dq, dk, dv};
    const void* ins[4] = {q, k, v, dout};
    for (int a = 0; a < 3; ++a) {
        for (int b = 0; b < 4; ++b)
            if (overlaps(outs[a], tb, ins[b], tb)) return LA_ERR_INVALID_ARGUMENT;
        for (int b = a + 1; b < 3; ++b)
            if (overlaps(outs[a], tb, outs[b], tb)) return LA_ERR_INVALID_ARGUMENT;
        if (dinit_state && overlaps(dinit_state, sb, outs[a], tb)) return LA_ERR_INVALID_ARGUMENT;
    }
    if (dinit_state && init_state && overlaps(dinit_state, sb, init_state, sb)) return LA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (dinit_state && cudaMemsetAsync(dinit_state, 0, sb, st) != cudaSuccess) return LA_ERR_CUDA;
        return LA_OK;
    }
    const BackwardLayout L = backward_layout(T, num_seqs, heads, d, B, dtype, decay != nullptr);
    if (decay && (overlaps(decay, (size_t)heads * 4, dq, tb) || overlaps(decay, (size_t)heads * 4, dk, tb) ||
                  overlaps(decay, (size_t)heads * 4, dv, tb)))
        return LA_ERR_INVALID_ARGUMENT;
    if (!workspace) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(workspace, 256)) return LA_ERR_MISALIGNED;
    if (workspace_bytes < L.total) return LA_ERR_WORKSPACE_TOO_SMALL;
    if (overlaps(workspace, L.total, dq, tb) || overlaps(workspace, L.total, dk, tb) ||
        overlaps(workspace, L.total, dv, tb) || (dinit_state && overlaps(workspace, L.total, dinit_state, sb)))
        return LA_ERR_INVALID_ARGUMENT;
    // the rates are read by every pass: none of the workspace's copies may land on them,
    // and the final dS0 scaling reads them while it writes dinit_state
    if (decay && (overlaps(workspace, L.total, decay, (size_t)heads * 4) ||
                  (dinit_state && overlaps(decay, (size_t)heads * 4, dinit_state, sb))))
        return LA_ERR_INVALID_ARGUMENT;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void *rk = ws + L.off_rk, *rq = ws + L.off_rq, *rdo = ws + L.off_rdo, *rv = ws + L.off_rv, *rout = ws + L.off_rout;
    float* s0t = reinterpret_cast<float*>(ws + L.off_s0t);
    void* pws = ws + L.off_pws;

    // dQ = prefill(dO, V, K) from S0^T
    if (init_state) {
        const dim3 grid((unsigned)(num_seqs * heads), (unsigned)((d + 31) / 32), (unsigned)((d + 31) / 32));
        la::transpose_states_kernel<<<grid, dim3(32, 8), 0, st>>>(init_state, s0t, d);
        note_launch();
        if ((s = cuda_check()) != LA_OK) return s;
    }
    auto fwd = [&](const void* a, const void* b, const void* c, void* out, const float* init) {
        return decay ? la_prefill_decay(a, b, c, out, cu_seqlens, num_seqs, T, heads, d, B, dtype, init, decay, nullptr,
                                        pws, L.pws, stream)
                     : la_prefill(a, b, c, out, cu_seqlens, num_seqs, T, heads, d, B, dtype, init, pws, L.pws, stream);
    };
    if ((s = fwd(dout, v, k, dq, init_state ? s0t : nullptr)) != LA_OK) return s;
    if (backward_in_place_order(dtype, d, B, num_seqs, heads, decay != nullptr)) {
        // dV_s = sum_{t >= s} (k_s . q_t) dO_t and dK_s = sum_{t >= s} (v_s . dO_t) q_t: the
        // anti-causal prefills of (K, Q, dO) and (V, dO, Q), in the tensors' own order
        const Layout PL = prefill_layout(T, num_seqs, heads, d, B, dtype);
        uint8_t* pw = static_cast<uint8_t*>(pws);
        if ((s = launch_chain(k, q, dout, dv, cu_seqlens, num_seqs, T, heads, d, B, nullptr, nullptr, pw, PL, st,
                              nullptr, true)) != LA_OK ||
            (s = launch_chain(v, dout, q, dk, cu_seqlens, num_seqs, T, heads, d, B, nullptr, nullptr, pw, PL, st,
                              nullptr, true)) != LA_OK)
            return s;
    } else {
    // dV and dK: forward prefills over the reversed sequences, reversed back
    if ((s = launch_reverse(k, rk, cu_seqlens, num_seqs, T, heads, d, dtype, st)) != LA_OK ||
        (s = launch_reverse(q, rq, cu_seqlens, num_seqs, T, heads, d, dtype, st)) != LA_OK ||
        (s = launch_reverse(dout, rdo, cu_seqlens, num_seqs, T, heads, d, dtype, st)) != LA_OK ||
        (s = launch_reverse(v, rv, cu_seqlens, num_seqs, T, heads, d, dtype, st)) != LA_OK)
        return s;
    if ((s = fwd(rk, rq, rdo, rout, nullptr)) != LA_OK ||
        (s = launch_reverse(rout, dv, cu_seqlens, num_seqs, T, heads, d, dtype, st)) != LA_OK)
        return s;
    if ((s = fwd(rv, rdo, rq, rout, nullptr)) != LA_OK ||
        (s = launch_reverse(rout, dk, cu_seqlens, num_seqs, T, heads, d, dtype, st)) != LA_OK)
        return s;
    }
    if (!dinit_state) return LA_OK;
    if (!decay)   // dS0 = state of (Q, dO)
        return la_state_from_prefill(q, dout, cu_seqlens, num_seqs, T, heads, d, dtype, nullptr, dinit_state,
                                     ws + L.off_sws, L.sws, stream);
    // decay: dS0 = lambda R_start, R_start = the decayed state of the reversed (Q, dO)
    if ((s = la_state_decay(rq, rdo, cu_seqlens, num_seqs, T, heads, d, dtype, nullptr, decay, dinit_state,
                            ws + L.off_sws, L.sws, stream)) != LA_OK)
        return s;
    const int sms = num_sms();
    if (sms <= 0) return LA_ERR_CUDA;
    const int64_t per_state4 = (int64_t)d * d / 4, total4 = (int64_t)num_seqs * heads * per_state4;
    const unsigned grid = (unsigned)std::min<int64_t>((total4 + 255) / 256, (int64_t)sms * 8);
    la::scale_states_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<float4*>(dinit_state), decay, heads, per_state4,
                                                 total4);
    note_launch();
    return cuda_check();
}

extern "C" {

// ---------------------------------------------------------------- decay variant
size_t la_prefill_decay_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, int B, la_dtype dtype) {
    if (total_tokens < 0 || num_seqs < 1 || heads < 1 || !supported_d(d) || !supported_B(B) ||
        (dtype != LA_BF16 && dtype != LA_FP32))
        return 0;
    if (total_tokens > 0 && prefill_path(dtype, d, B, num_seqs, heads) == Path::chain)
        return prefill_layout(total_tokens, num_seqs, heads, d, B, dtype).total;
    return simt_layout(total_tokens, num_seqs, heads, d, B).total;
}

la_status la_prefill_decay(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens,
                           int num_seqs, int64_t total_tokens, int heads, int d, int B, la_dtype dtype,
                           const float* init_state, const float* decay, float* state_out, void* workspace,
                           size_t workspace_bytes, void* stream) {
    la_status s = check_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state);
    if (s != LA_OK) return s;
    if (!decay) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(decay, 4)) return LA_ERR_MISALIGNED;
    const size_t tb = (size_t)total_tokens * heads * d * esize(dtype);
    const size_t sb = (size_t)num_seqs * heads * d * d * 4;
    const size_t db = (size_t)heads * 4;
    if (overlaps(decay, db, o, tb)) return LA_ERR_INVALID_ARGUMENT;
    if (state_out) {
        if (!aligned(state_out, 16)) return LA_ERR_MISALIGNED;
        // state_out may be init_state itself: the scan reads each element of S0 before it writes it
        if (init_state && init_state != state_out && overlaps(state_out, sb, init_state, sb))
            return LA_ERR_INVALID_ARGUMENT;
        if (overlaps(state_out, sb, o, tb) || overlaps(state_out, sb, q, tb) || overlaps(state_out, sb, k, tb) ||
            overlaps(state_out, sb, v, tb) || overlaps(state_out, sb, decay, db))
            return LA_ERR_INVALID_ARGUMENT;
    }
    if (total_tokens == 0 && !state_out) return LA_OK;
    // the on-chip-state tensor-core kernel where la_prefill would use it, else CUDA cores
    const bool chain = total_tokens > 0 && prefill_path(dtype, d, B, num_seqs, heads) == Path::chain;
    const Layout L = chain ? prefill_layout(total_tokens, num_seqs, heads, d, B, dtype)
                           : simt_layout(total_tokens, num_seqs, heads, d, B);
    if (!workspace) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(workspace, 256)) return LA_ERR_MISALIGNED;
    if (workspace_bytes < L.total) return LA_ERR_WORKSPACE_TOO_SMALL;
    if (overlaps(workspace, L.total, o, tb) || overlaps(workspace, L.total, decay, db) ||
        (state_out && overlaps(workspace, L.total, state_out, sb)))
        return LA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (chain)
        return launch_chain(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, init_state, state_out, ws, L,
                            st, decay);
    if ((s = launch_block_table(cu_seqlens, num_seqs, total_tokens, B, heads, L, ws, st)) != LA_OK) return s;
    if ((s = launch_decay_check(decay, heads, ws, st)) != LA_OK) return s;
    if (total_tokens > 0 && (s = simt_states_d(d, dtype, k, v, heads, L, ws, decay, st)) != LA_OK) return s;
    const int dd = d * d;
    dim3 sg((dd + 1023) / 1024, num_seqs * heads);
    la::chain_scan_kernel<float><<<sg, 256, 0, st>>>(
        reinterpret_cast<const float*>(ws + L.off_U), reinterpret_cast<float*>(ws + L.off_prefix), init_state,
        state_out, reinterpret_cast<const int32_t*>(ws + L.off_seq_blk), reinterpret_cast<const Control*>(ws),
        num_seqs, heads, dd, state_out == nullptr, reinterpret_cast<const BlockEntry*>(ws + L.off_table), decay);
    note_launch();
    if ((s = cuda_check()) != LA_OK) return s;
    if (total_tokens == 0) return LA_OK;
    MainKernelTimer timer(st);
    return simt_prefill_d(d, dtype, q, k, v, o, heads, B, L, ws, decay, st);
}

size_t la_state_decay_workspace_size(int64_t total_tokens, int num_seqs, int heads, int d, la_dtype dtype) {
    if (total_tokens < 0 || num_seqs < 1 || heads < 1 || !supported_d(d) || (dtype != LA_BF16 && dtype != LA_FP32))
        return 0;
    return simt_state_layout(total_tokens, num_seqs, heads, d).total;
}

la_status la_state_decay(const void* k, const void* v, const int32_t* cu_seqlens, int num_seqs,
                         int64_t total_tokens, int heads, int d, la_dtype dtype, const float* init_state,
                         const float* decay, float* state_out, void* workspace, size_t workspace_bytes,
                         void* stream) {
    la_status s = check_tokens(total_tokens, num_seqs, heads, d, dtype, cu_seqlens);
    if (s != LA_OK) return s;
    if (!state_out || !decay || (total_tokens > 0 && (!k || !v))) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(state_out, 16) || !aligned(decay, 4)) return LA_ERR_MISALIGNED;
    if (init_state && !aligned(init_state, 16)) return LA_ERR_MISALIGNED;
    const size_t sb = (size_t)num_seqs * heads * d * d * 4;
    const size_t tb = (size_t)total_tokens * heads * d * esize(dtype);
    if (init_state && init_state != state_out && overlaps(init_state, sb, state_out, sb)) return LA_ERR_INVALID_ARGUMENT;
    if (overlaps(state_out, sb, k, tb) || overlaps(state_out, sb, v, tb) || overlaps(state_out, sb, decay, heads * 4))
        return LA_ERR_INVALID_ARGUMENT;
    const Layout L = simt_state_layout(total_tokens, num_seqs, heads, d);
    if (!workspace) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(workspace, 256)) return LA_ERR_MISALIGNED;
    if (workspace_bytes < L.total) return LA_ERR_WORKSPACE_TOO_SMALL;
    if (overlaps(workspace, L.total, state_out, sb)) return LA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if ((s = launch_block_table(cu_seqlens, num_seqs, total_tokens, kStateBlock, heads, L, ws, st)) != LA_OK) return s;
    if ((s = launch_decay_check(decay, heads, ws, st)) != LA_OK) return s;
    if (total_tokens > 0 && (s = simt_states_d(d, dtype, k, v, heads, L, ws, decay, st)) != LA_OK) return s;
    const int dd = d * d;
    dim3 sg((dd + 1023) / 1024, num_seqs * heads);
    la::chain_scan_kernel<float><<<sg, 256, 0, st>>>(
        reinterpret_cast<const float*>(ws + L.off_U), static_cast<float*>(nullptr), init_state, state_out,
        reinterpret_cast<const int32_t*>(ws + L.off_seq_blk), reinterpret_cast<const Control*>(ws), num_seqs,
        heads, dd, false, reinterpret_cast<const BlockEntry*>(ws + L.off_table), decay);
    note_launch();
    return cuda_check();
}

la_status la_decode_step_decay(const void* q, const void* k, const void* v, float* state, void* o, int batch,
                               int heads, int d, la_dtype dtype, const float* decay, void* stream) {
    if (batch < 0 || heads < 1) return LA_ERR_INVALID_ARGUMENT;
    if (dtype != LA_BF16 && dtype != LA_FP32) return LA_ERR_UNSUPPORTED;
    if (!supported_d(d)) return LA_ERR_UNSUPPORTED;
    if (batch == 0) return LA_OK;
    if (!q || !k || !v || !state || !o || !decay) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(state, 16) ||
        !aligned(decay, 4))
        return LA_ERR_MISALIGNED;
    const int64_t pairs = (int64_t)batch * heads;
    const size_t vec = (size_t)pairs * d * esize(dtype);
    const size_t sbytes = (size_t)pairs * d * d * 4;
    const size_t db = (size_t)heads * 4;
    if (overlaps(o, vec, q, vec) || overlaps(o, vec, k, vec) || overlaps(o, vec, v, vec) ||
        overlaps(o, vec, state, sbytes) || overlaps(state, sbytes, q, vec) || overlaps(state, sbytes, k, vec) ||
        overlaps(state, sbytes, v, vec) || overlaps(decay, db, state, sbytes) || overlaps(decay, db, o, vec))
        return LA_ERR_INVALID_ARGUMENT;
    if (pairs >= (int64_t(1) << 31)) return LA_ERR_UNSUPPORTED;
    MainKernelTimer timer(reinterpret_cast<cudaStream_t>(stream));
    return decode_d(d, dtype, q, k, v, state, o, pairs, decay, heads, reinterpret_cast<cudaStream_t>(stream));
}

la_status la_feature_map(const void* x, void* y, int64_t n, la_dtype dtype, float alpha, void* stream) {
    if (n < 0) return LA_ERR_INVALID_ARGUMENT;
    if (dtype != LA_BF16 && dtype != LA_FP32) return LA_ERR_UNSUPPORTED;
    if (!(alpha == alpha) || alpha > 3.4e38f || alpha < -3.4e38f) return LA_ERR_INVALID_ARGUMENT;
    if (n == 0) return LA_OK;
    if (!x || !y) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(x, 16) || !aligned(y, 16)) return LA_ERR_MISALIGNED;
    const size_t bytes = (size_t)n * esize(dtype);
    if (x != y && overlaps(x, bytes, y, bytes)) return LA_ERR_INVALID_ARGUMENT;
    const int sms = num_sms();
    if (sms <= 0) return LA_ERR_CUDA;
    const int64_t groups = n / (16 / (int64_t)esize(dtype));
    const int64_t want = std::max<int64_t>(1, (groups + 255) / 256);
    const unsigned grid = (unsigned)std::min<int64_t>(want, (int64_t)sms * 8);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == LA_BF16)
        la::feature_map_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), n, alpha);
    else
        la::feature_map_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), static_cast<float*>(y), n,
                                                             alpha);
    note_launch();
    return cuda_check();
}

la_status la_get_device_status(void* stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return LA_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, la::g_status, sizeof(int)) != cudaSuccess) return LA_ERR_CUDA;
    if (cudaMemcpyToSymbol(la::g_status, &zero, sizeof(int)) != cudaSuccess) return LA_ERR_CUDA;
    return static_cast<la_status>(v);
}

la_status la_debug_set_fault(long long suppress_tile, uint64_t wait_ns) {
    if (suppress_tile < -1) return LA_ERR_INVALID_ARGUMENT;
    t_suppress_tile = suppress_tile;
    t_wait_ns = wait_ns;
    return LA_OK;
}

uint64_t la_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

la_status la_debug_set_path(int path) {
    if (path < 0 || path > 2) return LA_ERR_INVALID_ARGUMENT;
    t_force_path = path;
    return LA_OK;
}

la_status la_debug_set_trace(void* device_buffer, size_t bytes) {
    if ((device_buffer == nullptr) != (bytes == 0)) return LA_ERR_INVALID_ARGUMENT;
    if (device_buffer && !aligned(device_buffer, 8)) return LA_ERR_MISALIGNED;
    t_trace = static_cast<uint64_t*>(device_buffer);
    t_trace_bytes = bytes;
    return LA_OK;
}

la_status la_set_kernel_timer(void* start_event, void* stop_event) {
    if ((start_event == nullptr) != (stop_event == nullptr)) return LA_ERR_INVALID_ARGUMENT;
    t_timer_start = reinterpret_cast<cudaEvent_t>(start_event);
    t_timer_stop = reinterpret_cast<cudaEvent_t>(stop_event);
    return LA_OK;
}

const char* la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "ok";
        case LA_ERR_INVALID_ARGUMENT: return "invalid argument";
        case LA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case LA_ERR_MISALIGNED: return "pointer not 16-byte aligned (workspace: 256-byte)";
        case LA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case LA_ERR_CUDA: return "CUDA error";
        case LA_ERR_TIMEOUT: return "device-side wait timed out";
        case LA_ERR_BAD_SEQLENS: return "cu_seqlens inconsistent with total_tokens";
        case LA_ERR_BAD_DECAY: return "a decay rate outside [0, 1]";
    }
    return "unknown status";
}

int la_version(void) { return 100; }

}  // extern "C"
