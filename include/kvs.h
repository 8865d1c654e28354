/*
 * kvs.h -- C ABI of the KV-streams hot path on NVIDIA B200 (sm_100a).
 *
 * KV-streams keeps generating from a KV cache that is compacted in place
 * instead of re-prefilled, and trains on the continuous trace with an
 * attention mask that reproduces the evictions. Sources (page title, section):
 *   [T]  "KV-streams: speeding up agentic RL by operating on the KV cache
 *        directly" (thread): the two fixes (logical RoPE positions kept apart
 *        from physical slots; whole 16-token blocks removed and block-table
 *        references joined), 1-token blocks in the SGLang setup, recorded
 *        compaction events replayed by the trainer.
 *   [P]  "KV-streams for Efficient Compaction in Agentic Reinforcement
 *        Learning" (paper listing): abstract; Fig. 2(A) (continuous trace with
 *        an attention mask that reproduces eviction).
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller, unless a
 *    parameter says "host". The library allocates no memory and keeps no
 *    state between calls; scratch space is passed in as `ws` of the size the
 *    matching *_ws_bytes() query returns. The one exception is
 *    kvs_paged_decode_attn_static: its scratch is a fixed 16 MiB array in the
 *    library's device image, and it caches that array's device address per
 *    device and CUDA context (see its comment).
 *  - Every call is asynchronous on `stream`, except kvs_build_tile_mask, which
 *    synchronises `stream` once to learn the sizes of its outputs
 *    (kvs_build_tile_mask_async is its asynchronous form).
 *  - Errors the host can see (NULL or misaligned pointers, bad sizes,
 *    unsupported dtype/head size) are returned at once and nothing is
 *    launched. Errors that depend on device data are written to `*dev_status`
 *    (an int32 the caller zeroes; first error wins, later calls do not clear
 *    it); kernels never trap. `dev_status` may be NULL, in which case such
 *    errors are not reported (the kernels still skip the offending work).
 *  - Tensors are contiguous, row-major, in the layouts listed per call.
 *  - Event convention: kvs_evict_range {seq, tau, start, end} removes logical
 *    positions [start, end) of sequence `seq` before the token at logical
 *    position `tau` is generated. A query at logical position t therefore may
 *    see key j iff j <= t < kappa_j, where kappa_j is the smallest tau of the
 *    events covering j ([T], trainer replay; [P] Fig. 2(A)).
 */
#ifndef KVS_H_
#define KVS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kvs_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    KVS_OK = 0,
    KVS_ERR_INVALID_ARG = 1, /* bad pointer, size, or out-of-range block id / slot   */
    KVS_ERR_UNALIGNED = 2,   /* eviction range covers part of a block (or the tail)  */
    KVS_ERR_EVENT_ORDER = 3, /* events not sorted by (seq, tau, start), or end > tau */
    KVS_ERR_CAPACITY = 4,    /* caller's output buffer too small / size limit        */
    KVS_ERR_UNSUPPORTED = 5, /* dtype / head size combination not built              */
    KVS_ERR_TIMEOUT = 6,     /* a bounded device wait gave up (kernel returned)      */
    KVS_ERR_CUDA = 7         /* a CUDA runtime call failed                           */
} kvs_status;

typedef enum { KVS_F32 = 0, KVS_BF16 = 1 } kvs_dtype;

/* One compaction event: logical positions [start, end) of sequence `seq`
 * removed before the token at logical position `tau` is generated. Inference
 * logs one such record per eviction and the trainer replays the log ([T],
 * trainer replay). Requires 0 <= start < end <= tau. */
typedef struct {
    int32_t seq, tau, start, end;
} kvs_evict_range;

enum { KVS_TILE_EMPTY = 0, KVS_TILE_FULL = 1, KVS_TILE_PARTIAL = 2 };

/*
 * Compiled eviction mask for B traces of N logical tokens, T = ceil(N/128).
 * Tile (b, qi, kj) covers queries [128qi, 128qi+128) x keys [128kj, 128kj+128).
 * It is EMPTY if none of its pairs is visible, FULL if all are (pairs past N
 * are not visible), PARTIAL otherwise.
 *   kappa    int32 [B][N]      first event time removing each key (INT32_MAX: never)
 *   cls      uint8 [B][T][T]   tile class
 *   row_ptr  int32 [B*T + 1]   row-CSR over (b, qi); row_col: kj ascending;
 *   row_col, row_pidx int32 [nnz]   row_pidx: partial index or -1 for FULL
 *   col_ptr  int32 [B*T + 1]   col-CSR over (b, kj); col_row: qi ascending;
 *   col_row, col_pidx int32 [nnz]   col_pidx: same partial index as the row entry
 *   bits     uint32 [n_partial][128][4]  bit (c % 32) of word (c / 32) of row r
 *            is set iff query 128qi + r sees key 128kj + c. Partial tiles are
 *            numbered in row-CSR order.
 * nnz_cap / partial_cap give the capacity (entries / tiles) of the list and
 * bits buffers. All pointers are device pointers.
 */
typedef struct {
    int32_t *kappa;
    uint8_t *cls;
    int32_t *row_ptr, *row_col, *row_pidx;
    int32_t *col_ptr, *col_row, *col_pidx;
    uint32_t *bits;
    int64_t nnz_cap, partial_cap;
    int32_t B, N, T;
} kvs_tile_mask;

typedef struct {
    int64_t nnz;       /* non-empty tiles */
    int64_t n_partial; /* partial tiles   */
    int64_t visible_pairs; /* unmasked (query, key) pairs, summed over traces */
} kvs_mask_sizes;

/*
 * Compile the compaction-event log into the tile mask ([T] trainer replay;
 * [P] Fig. 2(A)).
 *   ev      device kvs_evict_range[n_ev], sorted by (seq, tau, start)
 *   m       host struct of device pointers; m->B, m->N must equal B, N.
 *           m->kappa, m->cls, m->row_ptr, m->col_ptr are always written.
 *           If m->row_col is NULL the call only counts (sizes out, lists
 *           untouched); otherwise the lists and bits are written when they fit
 *           (nnz <= nnz_cap, n_partial <= partial_cap), else KVS_ERR_CAPACITY.
 *   sizes   host out: nnz, n_partial, visible_pairs (always filled on KVS_OK
 *           and on KVS_ERR_CAPACITY).
 *   ws      device scratch of kvs_build_tile_mask_ws_bytes(B, N) bytes.
 * Synchronises `stream` once (after counting). Event-log errors
 * (KVS_ERR_EVENT_ORDER, KVS_ERR_INVALID_ARG for seq out of range) are returned.
 */
size_t kvs_build_tile_mask_ws_bytes(int32_t B, int32_t N);
kvs_status kvs_build_tile_mask(const kvs_evict_range *ev, int32_t n_ev, int32_t B, int32_t N,
                               kvs_tile_mask *m, kvs_mask_sizes *sizes, void *ws, size_t ws_bytes,
                               kvs_stream_t stream);

/*
 * The same compilation ([T] trainer replay; [P] Fig. 2(A)) without the host
 * round trip, for a training loop that keeps the mask buffers from step to
 * step: nothing is read back and `stream` is never synchronised, so the call
 * neither stalls the host nor waits behind other device-to-host copies.
 *   m          as above, with every list pointer set (bits may be NULL only
 *              when partial_cap == 0) and nnz_cap / partial_cap the capacity
 *              of the buffers, e.g. from a counting call on the same log or a
 *              bound the caller derives.
 *   dev_sizes  device int64 [3] or NULL: nnz, n_partial, visible_pairs.
 *   dev_status device int32 (first error wins) or NULL.
 * Event-log errors (as above) and lists over capacity (KVS_ERR_CAPACITY) are
 * written to *dev_status; the lists are then not written and every row_ptr and
 * col_ptr entry is set to 0, so the mask reads as empty: an attention call made
 * on it anyway loads no tile, and its outputs carry no meaning. Host-visible
 * argument errors are returned at once and nothing is launched.
 */
kvs_status kvs_build_tile_mask_async(const kvs_evict_range *ev, int32_t n_ev, int32_t B, int32_t N,
                                     kvs_tile_mask *m, int64_t *dev_sizes, void *ws, size_t ws_bytes,
                                     int32_t *dev_status, kvs_stream_t stream);

/*
 * Block-table compaction ([T] second fix: only whole blocks leave the cache,
 * and the surviving references are packed together so the table has no
 * holes). In place, per sequence b:
 * every live entry i < num_blocks[b] whose logical span
 * [block_lpos[b][i], block_lpos[b][i] + block_size) lies inside one of the
 * sequence's ranges is removed; the others keep their order and move down;
 * removed block ids are written, in table order, to freed[b][0..n_freed[b]);
 * entries past the new count are set to -1; num_tokens[b] drops by
 * block_size per removed block.
 *   block_table, block_lpos, freed  int32 [B][max_blocks]
 *   num_blocks, num_tokens, n_freed int32 [B]
 *   ev      device kvs_evict_range[n_ev] sorted by seq (tau is not used here)
 * A range that covers only part of a block, or any part of a partly filled
 * tail block (num_tokens % block_size != 0), sets KVS_ERR_UNALIGNED; a block
 * id outside [0, pool_blocks) sets KVS_ERR_INVALID_ARG; in both cases that
 * sequence is left unchanged and n_freed[b] = 0. A range covering positions
 * removed earlier is legal.
 */
kvs_status kvs_compact_block_table(int32_t *block_table, int32_t *block_lpos, int32_t *num_blocks,
                                   int32_t *num_tokens, int32_t B, int32_t max_blocks,
                                   int32_t block_size, int32_t pool_blocks,
                                   const kvs_evict_range *ev, int32_t n_ev, int32_t *freed,
                                   int32_t *n_freed, int32_t *dev_status, kvs_stream_t stream);

/*
 * Rotary embedding at LOGICAL positions ([T] first fix: cached keys keep the
 * rotation of their original position; new queries and keys continue the
 * original position count). Rotate-half convention: for i < d/2,
 *   (x_i, x_{i+d/2}) -> (x_i c - x_{i+d/2} s, x_i s + x_{i+d/2} c),
 *   angle = p * theta^(-2i/d), p = lpos[n] (or -lpos[n] if inverse != 0,
 *   which is the transpose, used for gradients). Angles in fp64, rotation
 *   in fp32.
 *   x       [n_tok] rows of H*d elements; row n starts at x + n*x_tok_stride
 *           (elements; heads contiguous within a row)
 *   lpos    int32 [n_tok]
 *   out_slot NULL: y is [n_tok][H][d] contiguous (block_size and
 *           pool_blocks are ignored).
 *           non-NULL (int64 [n_tok]): y is a paged cache
 *           [pool_blocks][H][block_size][d] and row n goes to slot out_slot[n]
 *           (block slot/bs, offset slot%bs); then, if v != NULL, v rows (same
 *           stride rules, v_tok_stride) are copied unrotated to the same slots
 *           of v_out (the value cache, same shape). A slot outside
 *           [0, pool_blocks * block_size) sets KVS_ERR_INVALID_ARG in
 *           *dev_status and its row is skipped: nothing is written for it.
 *   dt      KVS_BF16 or KVS_F32 for x, y, v, v_out; d in {64, 128}.
 */
kvs_status kvs_rope_logical(const void *x, int64_t x_tok_stride, void *y, const int32_t *lpos,
                            int32_t n_tok, int32_t H, int32_t d, double theta, int32_t inverse,
                            const int64_t *out_slot, int32_t block_size, int32_t pool_blocks,
                            const void *v, int64_t v_tok_stride, void *v_out, kvs_dtype dt,
                            int32_t *dev_status, kvs_stream_t stream);

/*
 * One paged decode step over the compacted block table ([T] second fix; the
 * attention walks the block table, which has no holes). For every sequence b
 * and query head h:
 *   o[b][h] = sum_i softmax_i(scale * <q[b][h], K_i>) V_i
 * over live entries i < num_tokens[b]; entry i is offset i % block_size of
 * block block_table[b][i / block_size]. kv head = h / (Hq / Hkv).
 *   q, o     [B][Hq][d] (q already rotated at its logical position)
 *   k_cache, v_cache  [pool_blocks][Hkv][block_size][d]
 *   block_table int32 [B][max_blocks]; num_tokens int32 [B] (0 gives o = 0)
 *   max_blocks * block_size must fit in int32 (else KVS_ERR_CAPACITY).
 *   dt      KVS_BF16 with d = 128, or KVS_F32 with d = 64 (fp32 accumulation)
 *   ws      device scratch of kvs_paged_decode_ws_bytes(...) bytes; no
 *           initialisation needed. Work split: the live entries of unit
 *           (b, kv head) are cut into chunks of 16; the units' chunks are laid
 *           end to end and C = min(444, B*Hkv*ceil(max_blocks*block_size/16))
 *           CTAs (one wave of 148 SMs x 3) take equal consecutive shares of
 *           them, found on the device from num_tokens. Scratch = 8*(B+1) bytes
 *           of prefix counts (rounded up to 256) + (C + B*Hkv) partial results
 *           of G*(d+2) fp32. The call runs the split kernel and a merge kernel.
 *           The table's chunk count B*Hkv*ceil(max_blocks*block_size/16) must
 *           fit in int32 (else KVS_ERR_CAPACITY).
 * Errors found in device data set KVS_ERR_INVALID_ARG in *dev_status:
 *  - a block id outside [0, pool_blocks): none of its entries is read; they
 *    are left out of the softmax (as if evicted);
 *  - num_tokens[b] < 0 or > max_blocks * block_size: the count is clamped to
 *    that range.
 */
size_t kvs_paged_decode_ws_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t d, int32_t block_size,
                                 int32_t max_blocks);
kvs_status kvs_paged_decode_attn(const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *block_table, const int32_t *num_tokens, int32_t B,
                                 int32_t Hq, int32_t Hkv, int32_t d, int32_t block_size,
                                 int32_t max_blocks, int32_t pool_blocks, float scale,
                                 kvs_dtype dt, void *o, void *ws, size_t ws_bytes,
                                 int32_t *dev_status, kvs_stream_t stream);

/*
 * kvs_paged_decode_attn for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for users whose decode
 * path must not call cudaMalloc (CUDA-graph replay of generation steps, engines
 * whose pool allocator owns all device memory, embedders that only receive
 * input/output pointers). Same arguments and results as kvs_paged_decode_attn
 * minus ws/ws_bytes: the scratch is a fixed array of
 * KVS_DECODE_STATIC_SCRATCH_BYTES (16 MiB) compiled into the library, held in
 * the memory of every GPU that loads it until the process exits.
 *  - Returns KVS_ERR_CAPACITY (nothing launched) when the call needs more
 *    scratch than that, i.e. kvs_paged_decode_ws_bytes(...) > the maximum.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *    The address is cached with the id of the device's CUDA context; after
 *    the context is destroyed and rebuilt (cudaDeviceReset) the next call
 *    looks it up again, so that call too must come before any capture.
 *  - All calls share the array: calls whose kernels overlap on the GPU
 *    (unordered streams, concurrent threads) race and give wrong results.
 *  - Allocates nothing: no cudaMalloc/cudaFree, no allocating library call.
 */
#define KVS_DECODE_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
kvs_status kvs_paged_decode_attn_static(const void *q, const void *k_cache, const void *v_cache,
                                        const int32_t *block_table, const int32_t *num_tokens,
                                        int32_t B, int32_t Hq, int32_t Hkv, int32_t d,
                                        int32_t block_size, int32_t max_blocks,
                                        int32_t pool_blocks, float scale, kvs_dtype dt, void *o,
                                        int32_t *dev_status, kvs_stream_t stream);

/*
 * Eviction-masked causal attention forward over the continuous trace ([T]
 * trainer replay; [P] Fig. 2(A)):
 *   O_t = sum_{j visible from t} softmax_j(scale <q_t, k_j>) v_j,
 *   lse_t = ln sum_{j visible} exp(scale <q_t, k_j>)
 * using the compiled mask m (EMPTY tiles skipped, PARTIAL tiles bit-masked).
 *   q, o    [B][N][Hq][d];  k, v [B][N][Hkv][d];  lse fp32 [B][Hq][N]
 *   o_lo    optional (NULL to skip), bf16 only, same layout as o: the rounding
 *           residual bf16(O - o) of the bf16 output, so that o + o_lo carries
 *           about 16 significant bits of the fp32 result. Pass it to the
 *           backward, which then forms D_t = <dO_t, O_t> from o + o_lo instead
 *           of the rounded o (the dominant bf16 error of the gradients).
 *   dt      KVS_BF16 (d = 128; tcgen05 tensor cores, fp32 accumulation) or
 *           KVS_F32 (d in {64, 128}; fp32 CUDA cores)
 * Pointers of bf16 tensors must be 16-byte aligned.
 */
kvs_status kvs_masked_attn_fwd(const void *q, const void *k, const void *v, const kvs_tile_mask *m,
                               int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d,
                               float scale, kvs_dtype dt, void *o, void *o_lo, float *lse,
                               int32_t *dev_status, kvs_stream_t stream);

/*
 * Backward of kvs_masked_attn_fwd (textbook softmax-attention gradients):
 *   D_t = <dO_t, O_t>; P_tj = exp(scale <q_t,k_j> - lse_t) on visible pairs;
 *   dV_j = sum_t P_tj dO_t;  dS_tj = P_tj (<dO_t, v_j> - D_t);
 *   dQ_t = scale sum_j dS_tj k_j;  dK_j = scale sum_t dS_tj q_t;
 * dK, dV of a kv head sum over its Hq/Hkv query heads.
 *   o, dO, dq [B][N][Hq][d]; dk, dv [B][N][Hkv][d]; lse as returned by the forward.
 *   o_lo    optional residual written by the forward (NULL: D uses o alone).
 *   ws      device scratch of kvs_masked_attn_bwd_ws_bytes(...) bytes.
 *   stages  bitmask of the three kernels the backward consists of:
 *           KVS_BWD_PREP (D and lse rows into ws), KVS_BWD_DKDV, KVS_BWD_DQ;
 *           KVS_BWD_ALL runs all three in order. Running them in separate calls
 *           (same ws, PREP first) gives the same result; dq is only written by
 *           KVS_BWD_DQ, dk and dv only by KVS_BWD_DKDV. The fp32 path ignores
 *           the mask and always runs everything.
 * Results are deterministic (no atomics).
 */
enum { KVS_BWD_PREP = 1, KVS_BWD_DKDV = 2, KVS_BWD_DQ = 4, KVS_BWD_ALL = 7 };
size_t kvs_masked_attn_bwd_ws_bytes(int32_t B, int32_t N, int32_t Hq, int32_t Hkv, int32_t d,
                                    kvs_dtype dt);
kvs_status kvs_masked_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                               const void *o_lo, const void *dO, const float *lse, const kvs_tile_mask *m, int32_t B,
                               int32_t N, int32_t Hq, int32_t Hkv, int32_t d, float scale,
                               kvs_dtype dt, void *dq, void *dk, void *dv, void *ws,
                               size_t ws_bytes, int32_t stages, int32_t *dev_status,
                               kvs_stream_t stream);

/* Text of the last CUDA runtime error behind a KVS_ERR_CUDA returned to the
 * calling thread ("no error" if there was none); a static string. */
const char *kvs_last_cuda_error(void);

/* Human-readable name of a status code (static string). */
const char *kvs_status_str(kvs_status s);

/* Library version as major*10000 + minor*100 + patch. */
int32_t kvs_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KVS_H_ */
