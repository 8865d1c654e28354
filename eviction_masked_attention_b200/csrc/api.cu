// C-ABI entry points of the masked attention forward/backward and small
// utilities. Host-side argument checks happen here; the kernels live in
// attn_fwd_tc.cu, attn_bwd_tc.cu (bf16, tcgen05) and attn_simt.cu (fp32).
#include "common.cuh"

namespace kvs {
cudaError_t launch_fwd_tc(const void *q, const void *k, const void *v, const kvs_tile_mask &m,
                          int32_t Hq, int32_t Hkv, float scale, void *o, void *o_lo, float *lse,
                          int32_t *status, cudaStream_t s, bool *map_ok);
cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const void *o,
                          const void *o_lo, const void *dO, const float *lse, const kvs_tile_mask &m, int32_t Hq,
                          int32_t Hkv, float scale, void *dq, void *dk, void *dv, void *ws,
                          int32_t stages, int32_t *status, cudaStream_t s, bool *map_ok);
size_t bwd_tc_ws_bytes(int32_t B, int32_t N, int32_t Hq);
cudaError_t launch_fwd_simt(const float *q, const float *k, const float *v, const kvs_tile_mask &m,
                            int32_t Hq, int32_t Hkv, int32_t d, float scale, float *o, float *lse,
                            cudaStream_t s);
cudaError_t launch_bwd_simt(const float *q, const float *k, const float *v, const float *o,
                            const float *dO, const float *lse, const kvs_tile_mask &m, int32_t Hq,
                            int32_t Hkv, int32_t d, float scale, float *dq, float *dk, float *dv,
                            float *Drow, cudaStream_t s);
}  // namespace kvs

using namespace kvs;

static kvs_status check_attn_args(const kvs_tile_mask *m, int32_t B, int32_t N, int32_t Hq,
                                  int32_t Hkv, int32_t d, kvs_dtype dt) {
    if (!m || B <= 0 || N <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return KVS_ERR_INVALID_ARG;
    if (m->B != B || m->N != N || m->T != (N + 127) / 128) return KVS_ERR_INVALID_ARG;
    if (!m->row_ptr || !m->row_col || !m->row_pidx || !m->col_ptr || !m->col_row || !m->col_pidx ||
        !m->kappa)
        return KVS_ERR_INVALID_ARG;
    if (m->partial_cap > 0 && !m->bits) return KVS_ERR_INVALID_ARG;
    if ((uintptr_t)m->bits % 16) return KVS_ERR_INVALID_ARG;
    if (dt == KVS_BF16) {
        if (d != 128) return KVS_ERR_UNSUPPORTED;
    } else if (dt == KVS_F32) {
        if (d != 64 && d != 128) return KVS_ERR_UNSUPPORTED;
    } else {
        return KVS_ERR_UNSUPPORTED;
    }
    if ((int64_t)B * Hq * m->T >= (1ll << 31)) return KVS_ERR_CAPACITY;
    return KVS_OK;
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

extern "C" kvs_status kvs_masked_attn_fwd(const void *q, const void *k, const void *v,
                                          const kvs_tile_mask *m, int32_t B, int32_t N, int32_t Hq,
                                          int32_t Hkv, int32_t d, float scale, kvs_dtype dt,
                                          void *o, void *o_lo, float *lse, int32_t *dev_status,
                                          kvs_stream_t stream) {
    kvs_status st = check_attn_args(m, B, N, Hq, Hkv, d, dt);
    if (st != KVS_OK) return st;
    if (!q || !k || !v || !o || !lse) return KVS_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(o_lo))
        return KVS_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == KVS_BF16) {
        bool map_ok = false;
        e = launch_fwd_tc(q, k, v, *m, Hq, Hkv, scale, o, o_lo, lse, dev_status, s, &map_ok);
        if (!map_ok) return KVS_ERR_INVALID_ARG;
    } else {
        e = launch_fwd_simt((const float *)q, (const float *)k, (const float *)v, *m, Hq, Hkv, d,
                            scale, (float *)o, lse, s);
    }
    return cuda_status(e);
}

extern "C" size_t kvs_masked_attn_bwd_ws_bytes(int32_t B, int32_t N, int32_t Hq, int32_t Hkv,
                                               int32_t d, kvs_dtype dt) {
    (void)Hkv;
    (void)d;
    if (B <= 0 || N <= 0 || Hq <= 0) return 0;
    if (dt == KVS_BF16) return bwd_tc_ws_bytes(B, N, Hq);
    return (size_t)B * Hq * N * sizeof(float);
}

extern "C" kvs_status kvs_masked_attn_bwd(const void *q, const void *k, const void *v,
                                          const void *o, const void *o_lo, const void *dO,
                                          const float *lse,
                                          const kvs_tile_mask *m, int32_t B, int32_t N, int32_t Hq,
                                          int32_t Hkv, int32_t d, float scale, kvs_dtype dt,
                                          void *dq, void *dk, void *dv, void *ws, size_t ws_bytes,
                                          int32_t stages, int32_t *dev_status,
                                          kvs_stream_t stream) {
    kvs_status st = check_attn_args(m, B, N, Hq, Hkv, d, dt);
    if (st != KVS_OK) return st;
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv || !ws) return KVS_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(ws) || !aligned16(o_lo))
        return KVS_ERR_INVALID_ARG;
    if (ws_bytes < kvs_masked_attn_bwd_ws_bytes(B, N, Hq, Hkv, d, dt)) return KVS_ERR_CAPACITY;
    if (stages <= 0 || stages > KVS_BWD_ALL) return KVS_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == KVS_BF16) {
        bool map_ok = false;
        e = launch_bwd_tc(q, k, v, o, o_lo, dO, lse, *m, Hq, Hkv, scale, dq, dk, dv, ws, stages,
                          dev_status, s, &map_ok);
        if (!map_ok) return KVS_ERR_INVALID_ARG;
    } else {
        e = launch_bwd_simt((const float *)q, (const float *)k, (const float *)v, (const float *)o,
                            (const float *)dO, lse, *m, Hq, Hkv, d, scale, (float *)dq, (float *)dk,
                            (float *)dv, (float *)ws, s);
    }
    return cuda_status(e);
}

extern "C" const char *kvs_status_str(kvs_status s) {
    switch (s) {
        case KVS_OK: return "ok";
        case KVS_ERR_INVALID_ARG: return "invalid argument";
        case KVS_ERR_UNALIGNED: return "eviction range covers part of a block";
        case KVS_ERR_EVENT_ORDER: return "event log not sorted or range past its time";
        case KVS_ERR_CAPACITY: return "buffer too small or size limit exceeded";
        case KVS_ERR_UNSUPPORTED: return "unsupported dtype / head size";
        case KVS_ERR_TIMEOUT: return "device wait timed out";
        case KVS_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

extern "C" int32_t kvs_version(void) { return 100; }

thread_local const char *kvs::g_last_cuda_error = nullptr;

extern "C" const char *kvs_last_cuda_error(void) {
    return kvs::g_last_cuda_error ? kvs::g_last_cuda_error : "no error";
}
