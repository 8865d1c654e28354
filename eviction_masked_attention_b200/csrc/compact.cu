// In-place block-table compaction.
//
// "KV-streams: speeding up agentic RL by operating on the KV cache directly",
// second fix: the engine finds 16-token blocks through a block table, cannot
// leave empty entries in it, and therefore removes complete blocks and joins
// the remaining block references; turns are padded to whole blocks (1-token
// blocks need no padding).
//
// One CTA per sequence. Pass 1 checks every live entry (a range may cover a
// block wholly or not at all; block ids must be in the pool). Pass 2 is a
// stable stream compaction in chunks of blockDim entries: each chunk is read
// into registers, then written to positions <= its own, so in-place is safe.
#include "common.cuh"

namespace kvs {

constexpr int kCompactThreads = 256;

__device__ inline int32_t block_exclusive_scan(int32_t v, int32_t *sh, int32_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int32_t x = v;
    for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int32_t s = lane < nw ? sh[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < nw) sh[lane] = s;
    }
    __syncthreads();
    int32_t incl = x + (warp ? sh[warp - 1] : 0);
    total = sh[nw - 1];
    __syncthreads();
    return incl - v;
}

// 0 = keep, 1 = drop, 2 = a range covers part of this block
__device__ inline int block_fate(int32_t lp, int32_t bs, bool is_tail_partial,
                                 const kvs_evict_range *ev, int32_t e0, int32_t e1) {
    int fate = 0;
    const int64_t a = lp, z = (int64_t)lp + bs;
    for (int32_t e = e0; e < e1; ++e) {
        const int64_t s = ev[e].start, f = ev[e].end;
        const int64_t lo = a > s ? a : s, hi = z < f ? z : f;
        if (lo >= hi) continue;
        if (s <= a && z <= f && !is_tail_partial) fate = fate == 2 ? 2 : 1;
        else fate = 2;
    }
    return fate;
}

__global__ void __launch_bounds__(kCompactThreads)
    k_compact(int32_t *block_table, int32_t *block_lpos, int32_t *num_blocks, int32_t *num_tokens,
              int32_t max_blocks, int32_t bs, int32_t pool_blocks, const kvs_evict_range *ev,
              int32_t n_ev, int32_t *freed, int32_t *n_freed, int32_t *status) {
    __shared__ int32_t sh[32];
    __shared__ int32_t s_bad;
    const int32_t b = blockIdx.x;
    int32_t *bt = block_table + (int64_t)b * max_blocks;
    int32_t *bl = block_lpos + (int64_t)b * max_blocks;
    int32_t *fr = freed + (int64_t)b * max_blocks;
    const int32_t n = min(max(num_blocks[b], 0), max_blocks);
    const int32_t ntok = num_tokens[b];
    const bool tail_partial = (ntok % bs) != 0;
    // this sequence's events (sorted by seq)
    int32_t lo = 0, hi = n_ev;
    while (lo < hi) {
        int32_t mid = (lo + hi) >> 1;
        if (ev[mid].seq < b) lo = mid + 1; else hi = mid;
    }
    const int32_t e0 = lo;
    hi = n_ev;
    while (lo < hi) {
        int32_t mid = (lo + hi) >> 1;
        if (ev[mid].seq <= b) lo = mid + 1; else hi = mid;
    }
    const int32_t e1 = lo;
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x) {
        int32_t id = bt[i];
        if (id < 0 || id >= pool_blocks) atomicOr(&s_bad, 1);
        if (block_fate(bl[i], bs, tail_partial && i == n - 1, ev, e0, e1) == 2) atomicOr(&s_bad, 2);
    }
    for (int32_t e = e0 + threadIdx.x; e < e1; e += blockDim.x)
        if (ev[e].start >= ev[e].end) atomicOr(&s_bad, 4);
    __syncthreads();
    if (s_bad) {
        if (threadIdx.x == 0) {
            set_status(status, (s_bad & 1) ? KVS_ERR_INVALID_ARG
                                           : ((s_bad & 2) ? KVS_ERR_UNALIGNED : KVS_ERR_EVENT_ORDER));
            n_freed[b] = 0;
        }
        return;
    }
    int32_t kept = 0, dropped = 0;
    for (int32_t base = 0; base < n; base += blockDim.x) {
        const int32_t i = base + threadIdx.x;
        int32_t id = -1, lp = -1, keep = 0, drop = 0;
        if (i < n) {
            id = bt[i];
            lp = bl[i];
            drop = block_fate(lp, bs, false, ev, e0, e1) == 1;
            keep = !drop;
        }
        int32_t tk, td;
        const int32_t pk = block_exclusive_scan(keep, sh, tk);
        const int32_t pd = block_exclusive_scan(drop, sh, td);
        // every thread of the chunk has read its entry (the scans synchronise)
        if (keep) {
            bt[kept + pk] = id;
            bl[kept + pk] = lp;
        }
        if (drop) fr[dropped + pd] = id;
        kept += tk;
        dropped += td;
        __syncthreads();
    }
    for (int32_t i = kept + threadIdx.x; i < n; i += blockDim.x) {
        bt[i] = -1;
        bl[i] = -1;
    }
    if (threadIdx.x == 0) {
        num_blocks[b] = kept;
        num_tokens[b] = ntok - dropped * bs;
        n_freed[b] = dropped;
    }
}

}  // namespace kvs

using namespace kvs;

extern "C" kvs_status kvs_compact_block_table(int32_t *block_table, int32_t *block_lpos,
                                              int32_t *num_blocks, int32_t *num_tokens, int32_t B,
                                              int32_t max_blocks, int32_t block_size,
                                              int32_t pool_blocks, const kvs_evict_range *ev,
                                              int32_t n_ev, int32_t *freed, int32_t *n_freed,
                                              int32_t *dev_status, kvs_stream_t stream) {
    if (B < 0 || max_blocks <= 0 || block_size <= 0 || pool_blocks <= 0 || n_ev < 0)
        return KVS_ERR_INVALID_ARG;
    if (B == 0) return KVS_OK;
    if (!block_table || !block_lpos || !num_blocks || !num_tokens || !freed || !n_freed ||
        (n_ev > 0 && !ev))
        return KVS_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    k_compact<<<B, kCompactThreads, 0, s>>>(block_table, block_lpos, num_blocks, num_tokens,
                                           max_blocks, block_size, pool_blocks, ev, n_ev, freed,
                                           n_freed, dev_status);
    return cuda_status(cudaGetLastError());
}
