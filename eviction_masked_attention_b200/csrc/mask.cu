// Compaction-event log -> kill times -> 128x128 tile mask.
//
// Follows the trainer replay of "KV-streams: speeding up agentic RL by
// operating on the KV cache directly" (a query may not attend to a range that
// an eviction at or before its position removed; the states of retained tokens
// stay as they were) and Fig. 2(A) of "KV-streams for Efficient Compaction in
// Agentic Reinforcement Learning" (one continuous trace, masked to reproduce
// the evictions).
//
// Key j is visible from query t iff j <= t < kappa_j. Inside one tile the
// visible rows of a key column form one interval [lo, hi), which the kernels
// use to classify tiles and to emit the bit rows of partial tiles.
#include "common.cuh"

namespace kvs {

constexpr int32_t kInfTau = 0x7fffffff;

// ws layout (int32 unless noted)
struct MaskWs {
    int32_t *tile_pidx;  // [B*T*T] partial index of each tile, -1 otherwise
    int32_t *row_nnz;    // [B*T]
    int32_t *row_npart;  // [B*T]
    int32_t *row_poff;   // [B*T + 1] exclusive scan of row_npart
    int32_t *col_cnt;    // [B*T]
    int32_t *status;     // [1]
    unsigned long long *pairs;  // [1]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ inline size_t mask_ws_layout(int32_t B, int32_t N, MaskWs *w, char *base) {
    const int64_t T = (N + 127) / 128;
    const int64_t BT = (int64_t)B * T;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base ? base + off : nullptr;
        off += align256(bytes);
        return p;
    };
    char *p0 = take(sizeof(int32_t) * BT * T);
    char *p1 = take(sizeof(int32_t) * BT);
    char *p2 = take(sizeof(int32_t) * BT);
    char *p3 = take(sizeof(int32_t) * (BT + 1));
    char *p4 = take(sizeof(int32_t) * BT);
    char *p5 = take(sizeof(int32_t) * 4);
    char *p6 = take(sizeof(unsigned long long) * 2);
    if (w) {
        w->tile_pidx = (int32_t *)p0;
        w->row_nnz = (int32_t *)p1;
        w->row_npart = (int32_t *)p2;
        w->row_poff = (int32_t *)p3;
        w->col_cnt = (int32_t *)p4;
        w->status = (int32_t *)p5;
        w->pairs = (unsigned long long *)p6;
    }
    return off;
}

// Events must be sorted by (seq, tau, start) with 0 <= start < end <= tau.
__global__ void k_validate_events(const kvs_evict_range *ev, int32_t n_ev, int32_t B,
                                  int32_t *status) {
    int32_t e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n_ev) return;
    kvs_evict_range r = ev[e];
    if (r.seq < 0 || r.seq >= B) set_status(status, KVS_ERR_INVALID_ARG);
    if (r.start < 0 || r.start >= r.end || r.end > r.tau) set_status(status, KVS_ERR_EVENT_ORDER);
    if (e > 0) {
        kvs_evict_range p = ev[e - 1];
        bool ordered = p.seq < r.seq || (p.seq == r.seq && (p.tau < r.tau ||
                                                            (p.tau == r.tau && p.start <= r.start)));
        if (!ordered) set_status(status, KVS_ERR_EVENT_ORDER);
    }
}

// First index of sequence b in the sorted event log.
__device__ inline int32_t lower_bound_seq(const kvs_evict_range *ev, int32_t n_ev, int32_t b) {
    int32_t lo = 0, hi = n_ev;
    while (lo < hi) {
        int32_t mid = (lo + hi) >> 1;
        if (ev[mid].seq < b) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// kappa[b][j]: events of a sequence are sorted by tau, so the first covering
// event gives the minimum. Also accumulates the visible-pair count.
__global__ void k_kappa(const kvs_evict_range *ev, int32_t n_ev, int32_t B, int32_t N,
                        int32_t *kappa, unsigned long long *pairs) {
    int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    unsigned long long cnt = 0;
    if (idx < (int64_t)B * N) {
        int32_t b = (int32_t)(idx / N), j = (int32_t)(idx % N);
        int32_t e = lower_bound_seq(ev, n_ev, b);
        int32_t kap = kInfTau;
        for (; e < n_ev && ev[e].seq == b; ++e)
            if (ev[e].start <= j && j < ev[e].end) {
                kap = ev[e].tau;
                break;
            }
        kappa[idx] = kap;
        int32_t hi = kap < N ? kap : N;
        cnt = hi > j ? (unsigned long long)(hi - j) : 0ull;
    }
    for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if ((threadIdx.x & 31) == 0 && cnt) atomicAdd(pairs, cnt);
}

// Visible row interval [lo, hi) of key k inside query tile starting at q0.
__device__ inline void col_interval(int32_t k, int32_t kap, int32_t q0, int32_t N, int32_t &lo,
                                    int32_t &hi) {
    if (k >= N) {
        lo = 0;
        hi = 0;
        return;
    }
    int64_t l = (int64_t)k - q0;
    int64_t h = (int64_t)(kap < N ? kap : N) - q0;
    lo = (int32_t)(l < 0 ? 0 : (l > 128 ? 128 : l));
    hi = (int32_t)(h < 0 ? 0 : (h > 128 ? 128 : h));
}

// One CTA per tile row (b, qi); each warp classifies tiles kj <= qi in turn.
// Writes cls (all T columns), per-row counts and per-column counts.
__global__ void k_classify(const int32_t *__restrict__ kappa, int32_t B, int32_t N, int32_t T,
                           uint8_t *__restrict__ cls, int32_t *row_nnz, int32_t *row_npart,
                           int32_t *col_cnt) {
    const int32_t row = blockIdx.x;  // b*T + qi
    const int32_t b = row / T, qi = row % T, q0 = qi * 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    __shared__ int32_t s_nnz, s_part;
    if (threadIdx.x == 0) s_nnz = s_part = 0;
    __syncthreads();
    const int32_t *kap = kappa + (int64_t)b * N;
    uint8_t *crow = cls + (int64_t)row * T;
    for (int32_t kj = warp; kj < T; kj += nw) {
        uint8_t c = KVS_TILE_EMPTY;
        if (kj <= qi) {
            bool any = false, all = true;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int32_t k = kj * 128 + lane + 32 * i;
                int32_t lo, hi;
                col_interval(k, k < N ? kap[k] : 0, q0, N, lo, hi);
                any |= lo < hi;
                all &= (lo == 0 && hi == 128);
            }
            any = __any_sync(0xffffffffu, any);
            all = __all_sync(0xffffffffu, all);
            c = !any ? KVS_TILE_EMPTY : (all ? KVS_TILE_FULL : KVS_TILE_PARTIAL);
        }
        if (lane == 0) {
            crow[kj] = c;
            if (c != KVS_TILE_EMPTY) {
                atomicAdd(&s_nnz, 1);
                atomicAdd(&col_cnt[b * T + kj], 1);
            }
            if (c == KVS_TILE_PARTIAL) atomicAdd(&s_part, 1);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        row_nnz[row] = s_nnz;
        row_npart[row] = s_part;
    }
}

// Exclusive scan of n int32 values into out[0..n]; one CTA of 1024 threads
// per array (blockIdx.x selects the array).
__global__ void k_scan3(const int32_t *in0, int32_t *out0, const int32_t *in1, int32_t *out1,
                        const int32_t *in2, int32_t *out2, int32_t n) {
    const int32_t *in = blockIdx.x == 0 ? in0 : (blockIdx.x == 1 ? in1 : in2);
    int32_t *out = blockIdx.x == 0 ? out0 : (blockIdx.x == 1 ? out1 : out2);
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int32_t base = 0; base < n; base += 1024) {
        int32_t i = base + threadIdx.x;
        int32_t v = i < n ? in[i] : 0;
        int32_t x = v;
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int32_t s = warp_sums[lane];
            for (int o = 1; o < 32; o <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            warp_sums[lane] = s;
        }
        __syncthreads();
        int32_t incl = x + (warp ? warp_sums[warp - 1] : 0) + carry;
        if (i < n) out[i] = incl - v;
        __syncthreads();
        if (threadIdx.x == 1023) carry = incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) out[n] = carry;
}

// One warp per tile row: ordered compaction of the row's non-empty tiles into
// the row-CSR, partial numbering, and the 128x4 bit words of partial tiles.
__global__ void k_fill_rows(const int32_t *__restrict__ kappa, const uint8_t *__restrict__ cls,
                            int32_t B, int32_t N, int32_t T, const int32_t *__restrict__ row_ptr,
                            const int32_t *__restrict__ row_poff, int32_t *row_col,
                            int32_t *row_pidx, int32_t *tile_pidx, uint32_t *bits, int64_t nnz_cap,
                            int64_t partial_cap) {
    const int lane = threadIdx.x & 31;
    const int32_t row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= B * T) return;
    // lists that do not fit are not written at all (the asynchronous build has no host check)
    if (row_ptr[B * T] > nnz_cap || row_poff[B * T] > partial_cap) return;
    const int32_t b = row / T, qi = row % T, q0 = qi * 128;
    const int32_t *kap = kappa + (int64_t)b * N;
    const uint8_t *crow = cls + (int64_t)row * T;
    int32_t e = row_ptr[row], p = row_poff[row];
    const unsigned lt = (1u << lane) - 1u;
    for (int32_t base = 0; base < T; base += 32) {
        int32_t kj = base + lane;
        uint8_t c = kj < T ? crow[kj] : KVS_TILE_EMPTY;
        unsigned nz = __ballot_sync(0xffffffffu, c != KVS_TILE_EMPTY);
        unsigned pt = __ballot_sync(0xffffffffu, c == KVS_TILE_PARTIAL);
        int32_t my_e = e + __popc(nz & lt), my_p = p + __popc(pt & lt);
        if (kj < T) {
            int32_t pid = c == KVS_TILE_PARTIAL ? my_p : -1;
            tile_pidx[(int64_t)row * T + kj] = pid;
            if (c != KVS_TILE_EMPTY) {
                row_col[my_e] = kj;
                row_pidx[my_e] = pid;
            }
        }
        // bits for the partial tiles of this chunk, one tile at a time
        unsigned todo = pt;
        int32_t pp = p;
        while (todo) {
            int src = __ffs(todo) - 1;
            todo &= todo - 1;
            int32_t tkj = base + src;
            int32_t lo[4], hi[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                int32_t k = tkj * 128 + 32 * w + lane;
                col_interval(k, k < N ? kap[k] : 0, q0, N, lo[w], hi[w]);
            }
            uint32_t *tb = bits + (int64_t)pp * 512;
            for (int r0 = 0; r0 < 128; r0 += 32) {
                uint32_t mine[4];
#pragma unroll
                for (int w = 0; w < 4; ++w)
#pragma unroll 4
                    for (int rr = 0; rr < 32; ++rr) {
                        int r = r0 + rr;
                        unsigned word = __ballot_sync(0xffffffffu, lo[w] <= r && r < hi[w]);
                        if (rr == lane) mine[w] = word;
                    }
                uint4 v = make_uint4(mine[0], mine[1], mine[2], mine[3]);
                *reinterpret_cast<uint4 *>(tb + (r0 + lane) * 4) = v;
            }
            ++pp;
        }
        e += __popc(nz);
        p += __popc(pt);
    }
}

// One warp per tile column (b, kj): ordered list of non-empty qi >= kj.
__global__ void k_fill_cols(const uint8_t *__restrict__ cls, int32_t B, int32_t T,
                            const int32_t *__restrict__ col_ptr,
                            const int32_t *__restrict__ tile_pidx, int32_t *col_row,
                            int32_t *col_pidx, const int32_t *__restrict__ row_poff, int64_t nnz_cap,
                            int64_t partial_cap) {
    const int lane = threadIdx.x & 31;
    const int32_t col = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (col >= B * T) return;
    if (col_ptr[B * T] > nnz_cap || row_poff[B * T] > partial_cap) return;
    const int32_t b = col / T, kj = col % T;
    int32_t e = col_ptr[col];
    const unsigned lt = (1u << lane) - 1u;
    for (int32_t base = kj; base < T; base += 32) {
        int32_t qi = base + lane;
        int64_t id = ((int64_t)b * T + qi) * T + kj;
        uint8_t c = qi < T ? cls[id] : KVS_TILE_EMPTY;
        unsigned nz = __ballot_sync(0xffffffffu, c != KVS_TILE_EMPTY);
        if (c != KVS_TILE_EMPTY) {
            int32_t my = e + __popc(nz & lt);
            col_row[my] = qi;
            col_pidx[my] = tile_pidx[id];
        }
        e += __popc(nz);
    }
}

// Last step of the asynchronous build: report the sizes, and on an event-log
// error or lists over capacity record the status and leave the mask empty
// (every row and column list of length zero), so that an attention call that
// runs on it anyway reads nothing it should not.
__global__ void k_mask_finish(int32_t *row_ptr, int32_t *col_ptr, const int32_t *__restrict__ row_poff,
                              const int32_t *__restrict__ ev_status,
                              const unsigned long long *__restrict__ pairs, int32_t BT, int64_t nnz_cap,
                              int64_t partial_cap, int64_t *sizes, int32_t *status) {
    const int32_t nnz = row_ptr[BT], np = row_poff[BT], est = *ev_status;
    const bool over = nnz > nnz_cap || np > partial_cap;
    __syncthreads();  // every thread has read the totals before any clears them
    if (threadIdx.x == 0) {
        if (sizes) {
            sizes[0] = nnz;
            sizes[1] = np;
            sizes[2] = (int64_t)*pairs;
        }
        if (est) set_status(status, est);
        else if (over) set_status(status, KVS_ERR_CAPACITY);
    }
    if (est || over)
        for (int32_t i = threadIdx.x; i <= BT; i += blockDim.x) {
            row_ptr[i] = 0;
            col_ptr[i] = 0;
        }
}

}  // namespace kvs

using namespace kvs;

extern "C" size_t kvs_build_tile_mask_ws_bytes(int32_t B, int32_t N) {
    if (B <= 0 || N <= 0) return 0;
    return mask_ws_layout(B, N, nullptr, nullptr);
}

namespace {

// Host checks shared by both builds; fills *w from ws.
kvs_status mask_args(const kvs_evict_range *ev, int32_t n_ev, int32_t B, int32_t N, kvs_tile_mask *m,
                     void *ws, size_t ws_bytes, MaskWs *w) {
    if (!m || B <= 0 || N <= 0 || n_ev < 0 || (n_ev > 0 && !ev)) return KVS_ERR_INVALID_ARG;
    if (m->B != B || m->N != N) return KVS_ERR_INVALID_ARG;
    const int64_t T64 = (N + 127) / 128;
    if ((int64_t)B * T64 * T64 >= (1ll << 31)) return KVS_ERR_CAPACITY;
    m->T = (int32_t)T64;
    if (!m->kappa || !m->cls || !m->row_ptr || !m->col_ptr) return KVS_ERR_INVALID_ARG;
    if (!ws || ws_bytes < kvs_build_tile_mask_ws_bytes(B, N)) return KVS_ERR_CAPACITY;
    mask_ws_layout(B, N, w, (char *)ws);
    return KVS_OK;
}

// Event checks, kill times, tile classes and the three scans (row offsets,
// partial offsets, column offsets).
kvs_status mask_count(const kvs_evict_range *ev, int32_t n_ev, int32_t B, int32_t N,
                      const kvs_tile_mask *m, const MaskWs &w, cudaStream_t s) {
    const int32_t T = m->T, BT = B * T;
    cudaError_t ce;
    if ((ce = cudaMemsetAsync(w.col_cnt, 0, sizeof(int32_t) * BT, s)) != cudaSuccess ||
        (ce = cudaMemsetAsync(w.status, 0, sizeof(int32_t) * 4, s)) != cudaSuccess ||
        (ce = cudaMemsetAsync(w.pairs, 0, sizeof(unsigned long long) * 2, s)) != cudaSuccess)
        return cuda_status(ce);
    if (n_ev > 0) k_validate_events<<<(n_ev + 255) / 256, 256, 0, s>>>(ev, n_ev, B, w.status);
    int64_t nthreads = (int64_t)B * N;
    k_kappa<<<(unsigned)((nthreads + 255) / 256), 256, 0, s>>>(ev, n_ev, B, N, m->kappa, w.pairs);
    k_classify<<<BT, 256, 0, s>>>(m->kappa, B, N, T, m->cls, w.row_nnz, w.row_npart, w.col_cnt);
    k_scan3<<<3, 1024, 0, s>>>(w.row_nnz, m->row_ptr, w.row_npart, w.row_poff, w.col_cnt,
                               m->col_ptr, BT);
    return (ce = cudaGetLastError()) != cudaSuccess ? cuda_status(ce) : KVS_OK;
}

// Row and column lists and the bit rows of partial tiles, each kernel skipping
// all writes when the totals exceed the capacities.
kvs_status mask_fill(int32_t B, int32_t N, const kvs_tile_mask *m, const MaskWs &w, cudaStream_t s) {
    const int32_t T = m->T, BT = B * T;
    const int rows_per_cta = 8;
    k_fill_rows<<<(BT + rows_per_cta - 1) / rows_per_cta, 32 * rows_per_cta, 0, s>>>(
        m->kappa, m->cls, B, N, T, m->row_ptr, w.row_poff, m->row_col, m->row_pidx, w.tile_pidx,
        m->bits, m->nnz_cap, m->partial_cap);
    k_fill_cols<<<(BT + rows_per_cta - 1) / rows_per_cta, 32 * rows_per_cta, 0, s>>>(
        m->cls, B, T, m->col_ptr, w.tile_pidx, m->col_row, m->col_pidx, w.row_poff, m->nnz_cap,
        m->partial_cap);
    cudaError_t ce;
    return (ce = cudaGetLastError()) != cudaSuccess ? cuda_status(ce) : KVS_OK;
}

}  // namespace

extern "C" kvs_status kvs_build_tile_mask(const kvs_evict_range *ev, int32_t n_ev, int32_t B,
                                          int32_t N, kvs_tile_mask *m, kvs_mask_sizes *sizes,
                                          void *ws, size_t ws_bytes, kvs_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!sizes) return KVS_ERR_INVALID_ARG;
    MaskWs w;
    kvs_status st = mask_args(ev, n_ev, B, N, m, ws, ws_bytes, &w);
    if (st != KVS_OK) return st;
    if ((st = mask_count(ev, n_ev, B, N, m, w, s)) != KVS_OK) return st;
    const int32_t BT = B * m->T;
    cudaError_t ce;
    int32_t h_nnz = 0, h_np = 0, h_st = 0;
    unsigned long long h_pairs = 0;
    if ((ce = cudaMemcpyAsync(&h_nnz, m->row_ptr + BT, 4, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (ce = cudaMemcpyAsync(&h_np, w.row_poff + BT, 4, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (ce = cudaMemcpyAsync(&h_st, w.status, 4, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (ce = cudaMemcpyAsync(&h_pairs, w.pairs, 8, cudaMemcpyDeviceToHost, s)) != cudaSuccess)
        return cuda_status(ce);
    if ((ce = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_status(ce);
    if (h_st != 0) return (kvs_status)h_st;
    sizes->nnz = h_nnz;
    sizes->n_partial = h_np;
    sizes->visible_pairs = (int64_t)h_pairs;
    if (!m->row_col) return KVS_OK;
    if (!m->row_pidx || !m->col_row || !m->col_pidx || (h_np > 0 && !m->bits))
        return KVS_ERR_INVALID_ARG;
    if (h_nnz > m->nnz_cap || h_np > m->partial_cap) return KVS_ERR_CAPACITY;
    return mask_fill(B, N, m, w, s);
}

extern "C" kvs_status kvs_build_tile_mask_async(const kvs_evict_range *ev, int32_t n_ev, int32_t B,
                                                int32_t N, kvs_tile_mask *m, int64_t *dev_sizes,
                                                void *ws, size_t ws_bytes, int32_t *dev_status,
                                                kvs_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    MaskWs w;
    kvs_status st = mask_args(ev, n_ev, B, N, m, ws, ws_bytes, &w);
    if (st != KVS_OK) return st;
    if (!m->row_col || !m->row_pidx || !m->col_row || !m->col_pidx || m->nnz_cap < 0 ||
        m->partial_cap < 0 || (m->partial_cap > 0 && !m->bits))
        return KVS_ERR_INVALID_ARG;
    if ((st = mask_count(ev, n_ev, B, N, m, w, s)) != KVS_OK) return st;
    if ((st = mask_fill(B, N, m, w, s)) != KVS_OK) return st;
    k_mask_finish<<<1, 256, 0, s>>>(m->row_ptr, m->col_ptr, w.row_poff, w.status, w.pairs, B * m->T,
                                    m->nnz_cap, m->partial_cap, dev_sizes, dev_status);
    cudaError_t ce;
    return (ce = cudaGetLastError()) != cudaSuccess ? cuda_status(ce) : KVS_OK;
}
