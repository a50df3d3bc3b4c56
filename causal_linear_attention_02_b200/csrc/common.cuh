// Shared device-side definitions of the Lightning Attention library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lightning_attention.h"

namespace la {

// ------------------------------------------------------------------ status word
// One word per device (this translation unit is the whole library, so a plain
// __device__ variable is visible to every kernel). The first device-side
// failure wins; la_get_device_status reads and clears it.
__device__ int g_status;

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_status, 0, code);
}

// ------------------------------------------------------------------ block table
// One entry per block of B tokens of one sequence (blocks restart at every
// sequence start; the last block of a sequence may be short). Built on the
// device from cu_seqlens by build_block_table_kernel.
struct BlockEntry {
    int32_t seq;    // sequence index
    int32_t blk;    // block index within the sequence
    int32_t tok0;   // first token (global row in the packed [T][H][d] tensors)
    int32_t len;    // tokens in this block (1..B)
    int32_t last;   // 1 for the last block of its sequence (its state is never needed)
    int32_t slot0;  // first published-state slot of this sequence (single-pass prefill)
    int32_t pad[2];
};
static_assert(sizeof(BlockEntry) == 32, "block table entries are 32 bytes");

// One sequence of a packed batch (the on-chip-state prefill walks sequences).
struct SeqEntry {
    int32_t tok0;   // first token (global row in the packed [T][H][d] tensors)
    int32_t len;    // tokens
};
static_assert(sizeof(SeqEntry) == 8, "sequence entries are 8 bytes");

// Published-state ring slots per (sequence, head) of the single-pass prefill.
constexpr int kStateSlots = 6;

// Small control area at the start of every prefill / state workspace.
struct Control {
    int32_t nblocks;     // number of valid BlockEntry rows
    int32_t ok;          // 1 when cu_seqlens passed the device-side checks
    int32_t nslots;      // published-state slots used (single-pass prefill)
    int32_t abort;       // set by any CTA of the single-pass prefill whose bounded wait expired
    int32_t nmulti;      // sequences of two or more tokens; the processing order lists them first
    int32_t nsingle;     // one-token sequences, listed next (0 unless the order is sorted)
    int32_t ticket;      // next one-token (sequence, head) of the prefill with final states
    int32_t pad[57];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

// ------------------------------------------------------------------ conversions
template <typename T> struct io;
template <> struct io<float> {
    static __device__ __forceinline__ float ld(const float* p) { return *p; }
    static __device__ __forceinline__ void st(float* p, float x) { *p = x; }
};
template <> struct io<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

// bf16x2 packing: `lo` goes to the low half (lower address / even index).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

}  // namespace la
