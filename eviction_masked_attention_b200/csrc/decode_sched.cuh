// Work split of the paged decode: every CTA gets an equal share of all live
// entries of the step, whatever the sequence lengths.
//
// The live entries of unit u = (sequence b, kv head kvh), u = b * Hkv + kvh,
// are cut into chunks of 16 (a chunk is one block when blocks hold 16 tokens).
// Units are laid end to end in u order: unit u owns global chunks
// [cs(u), cs(u) + nch(b)) with cs(u) = Hkv * pre(b) + kvh * nch(b), where
// nch(b) = ceil(num_tokens[b] / 16) and pre(b) = nch(0) + ... + nch(b-1).
// With TC = Hkv * pre(B) chunks in all and C CTAs, CTA c takes the chunks
// [c TC / C, (c+1) TC / C) (integer division): the pieces of the one or more
// units that this range crosses. A piece that is a whole unit writes the
// unit's output; any other piece writes its partial softmax state
// (unnormalised output, max, sum per query head) to slot c + u, which is unique
// because consecutive units share at most one CTA. The merge kernel finds the
// CTAs of a unit's first and last chunk and folds their slots.
//
// num_tokens is device data, so the split is found on the device: each CTA
// scans the per-sequence chunk counts (one value per thread group), and CTA 0
// also stores pre(0..B) for the merge kernel. C is one wave of 148 SMs x 3
// CTAs (fewer when the table holds fewer chunks); a CTA walks its share in
// sub-pieces of at most 72 chunks (the block-table slice it stages in shared
// memory), carrying its softmax state across the sub-pieces of a unit.
#pragma once
#include "common.cuh"

namespace kvs {

constexpr int kDecChunk = 16;            // entries per chunk
constexpr int kDecMaxChunksPerCta = 72;  // chunks per staged sub-piece (1152 entries)
constexpr int kDecWave = 148 * 3;        // resident CTAs of the bf16 decode kernel
constexpr int kDecThreads = 128;         // both decode kernels

struct DecodePlan {
    int64_t ctas;      // C
    int64_t units;     // B * Hkv
    size_t pre_off;    // byte offset of pre[0..B] (int64) in ws
    size_t part_off;   // byte offset of the partials in ws
    size_t ws_bytes;
};

// C and the scratch layout, from the table's capacity only (host arithmetic).
inline DecodePlan decode_plan(int32_t B, int32_t Hq, int32_t Hkv, int32_t d, int32_t bs,
                              int32_t max_blocks) {
    DecodePlan p;
    const int64_t max_tok = (int64_t)max_blocks * bs;
    const int64_t mc = (max_tok + kDecChunk - 1) / kDecChunk;
    p.units = (int64_t)B * Hkv;
    const int64_t tc_max = p.units * mc;
    int64_t c = kDecWave;
    if (c > tc_max) c = tc_max;
    if (c < 1) c = 1;
    p.ctas = c;
    const int G = Hq / Hkv;
    p.pre_off = 0;
    p.part_off = ((size_t)(B + 1) * sizeof(int64_t) + 255) & ~(size_t)255;
    p.ws_bytes = p.part_off + (size_t)(p.ctas + p.units) * G * (d + 2) * sizeof(float);
    return p;
}

// Live-entry count of sequence b as the kernels use it: clamped to [0, cap].
__device__ __forceinline__ int32_t dec_ntok(const int32_t *num_tokens, int32_t b, int32_t cap) {
    return min(max(num_tokens[b], 0), cap);
}
__device__ __forceinline__ int32_t dec_nch(int32_t ntok) {
    return (ntok + kDecChunk - 1) / kDecChunk;
}

// CTA that holds global chunk x.
__device__ __forceinline__ int64_t dec_cta_of(int64_t x, int64_t tc, int64_t C) {
    return ((x + 1) * C - 1) / tc;
}

// Chunk counts fit in int32 (the host rejects tables with more than INT32_MAX
// chunks), so the device keeps chunk coordinates in 32 bits; only the products
// c * TC of the split need 64.
struct DecodeRange {
    int32_t x0, x1;   // this CTA's global chunks
    int32_t b0;       // sequence of chunk x0
    int32_t pre_b0;   // pre(b0)
};

// Block-wide (kDecThreads threads) scan of the chunk counts; returns this CTA's
// range (x0 == x1: nothing to do). CTA 0 writes pre(0..B) to pre_out and reports
// counts outside [0, cap]. Every thread of the block must call it.
__device__ __forceinline__ DecodeRange dec_locate(const int32_t *num_tokens, int32_t B, int32_t Hkv,
                                                  int32_t cap, int64_t C, int64_t *pre_out,
                                                  int32_t *status) {
    __shared__ int32_t s_warp[kDecThreads / 32];
    __shared__ int32_t s_pre, s_b;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (B + kDecThreads - 1) / kDecThreads;
    const int bl = min(B, tid * per), bh = min(B, bl + per);
    int32_t loc = 0;
    for (int b = bl; b < bh; ++b) {
        const int32_t raw = num_tokens[b];
        if (blockIdx.x == 0 && (raw < 0 || raw > cap)) set_status(status, KVS_ERR_INVALID_ARG);
        loc += dec_nch(min(max(raw, 0), cap));
    }
    // exclusive scan of loc over the block
    int32_t inc = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_warp[warp] = inc;
    if (tid == 0) s_b = -1;
    __syncthreads();
    int32_t base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kDecThreads / 32; ++w) {
        if (w < warp) base += s_warp[w];
        tot += s_warp[w];
    }
    const int32_t excl = base + inc - loc;
    const int64_t tc = (int64_t)tot * Hkv;
    const int64_t c = blockIdx.x;
    DecodeRange r;
    r.x0 = (int32_t)(tc ? c * tc / C : 0);
    r.x1 = (int32_t)(tc ? (c + 1) * tc / C : 0);
    int32_t p = excl;
    for (int b = bl; b < bh; ++b) {
        const int32_t n = dec_nch(dec_ntok(num_tokens, b, cap));
        if (pre_out && blockIdx.x == 0) pre_out[b] = p;
        if (r.x0 < r.x1 && Hkv * p <= r.x0 && r.x0 < Hkv * (p + n)) {
            s_b = b;
            s_pre = p;
        }
        p += n;
    }
    if (pre_out && blockIdx.x == 0 && tid == kDecThreads - 1) pre_out[B] = tot;
    __syncthreads();
    r.b0 = s_b;
    r.pre_b0 = s_pre;
    if (r.b0 < 0) r.x1 = r.x0;  // empty range
    return r;
}

}  // namespace kvs
