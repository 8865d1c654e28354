// bf16 eviction-masked attention forward on sm_100a tensor cores.
//
// Replays the continuous trace with the eviction mask ("KV-streams: speeding
// up agentic RL by operating on the KV cache directly", trainer replay;
// "KV-streams for Efficient Compaction in Agentic Reinforcement Learning",
// Fig. 2(A)). Only the non-empty 128x128 tiles of the compiled mask are
// visited (row-CSR); PARTIAL tiles are bit-masked, FULL tiles are not.
//
// One CTA per (query tile, head, trace), 6 warps:
//   warp 0      TMA producer: Q once, then K and V tiles (2-stage rings each)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2..5  softmax: thread = TMEM lane = query row
// TMEM (512 columns): S double buffer [0,128) [128,256), O accumulator [256,384).
// Per tile n: S_n = Q K_n^T (SS MMA) -> softmax reads S_n, writes P_n as bf16
// into the first 64 columns of the same buffer -> O += P_n V_n (A operand from
// TMEM). S_{n+1} is issued before PV_n, so the tensor core works on the next
// scores while the softmax warps handle the current ones. The running max is
// only raised (and O rescaled in TMEM) when it grows by more than 2^8;
// otherwise the stale max stays exact because O and the row sum share it.
#include "common.cuh"

namespace kvs {

constexpr int kFwdThreads = 192;
constexpr uint32_t kTileBytes = 128 * 128 * 2;  // one 128x128 bf16 tile
constexpr float kRescaleThreshold = 8.0f;       // log2 units

struct FwdSmem {
    uint8_t q[kTileBytes];
    uint8_t k[2][kTileBytes];
    uint8_t v[2][kTileBytes];
    uint64_t bar_q, kfull[2], kempty[2], vfull[2], vempty[2], sfull[2], pfull[2], odone, fin;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool wait_final(uint64_t *bar, uint32_t parity) {
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

__global__ void __launch_bounds__(kFwdThreads, 1)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, kvs_tile_mask m, int32_t Hq,
                  int32_t Hkv, float scale_log2, __nv_bfloat16 *__restrict__ out,
                  float *__restrict__ lse, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem &S = *reinterpret_cast<FwdSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = m.B, N = m.N, T = m.T, G = Hq / Hkv;
    // heaviest tile rows (largest qi) first
    const int64_t idx = blockIdx.x;
    const int qi = T - 1 - (int)(idx / ((int64_t)B * Hq));
    const int rem = (int)(idx % ((int64_t)B * Hq));
    const int hq = rem % Hq, b = rem / Hq, kvh = hq / G;
    const int q0 = qi * 128;
    const int32_t e0 = m.row_ptr[b * T + qi], nt = m.row_ptr[b * T + qi + 1] - e0;
    if (grid_timed_out(status)) return;

    if (threadIdx.x == 0) {
        mbar_init(&S.bar_q, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.kfull[i], 1);
            mbar_init(&S.kempty[i], 1);
            mbar_init(&S.vfull[i], 1);
            mbar_init(&S.vempty[i], 1);
            mbar_init(&S.sfull[i], 1);
            mbar_init(&S.pfull[i], 128);
        }
        mbar_init(&S.odone, 1);
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    volatile int *abort = &S.abort;

    if (warp == 0) {
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_expect_tx(&S.bar_q, kTileBytes);
            tma_load_4d(S.q, &tmQ, &S.bar_q, 0, hq, q0, b);
            tma_load_4d(S.q + kTileBytes / 2, &tmQ, &S.bar_q, 64, hq, q0, b);
            for (int n = 0; n < nt; ++n) {
                const int s = n & 1;
                const uint32_t ph = ((n >> 1) - 1) & 1;
                const int k0 = m.row_col[e0 + n] * 128;
                if (n >= 2 && !mbar_wait(&S.kempty[s], ph, abort, status)) break;
                mbar_expect_tx(&S.kfull[s], kTileBytes);
                tma_load_4d(S.k[s], &tmK, &S.kfull[s], 0, kvh, k0, b);
                tma_load_4d(S.k[s] + kTileBytes / 2, &tmK, &S.kfull[s], 64, kvh, k0, b);
                if (n >= 2 && !mbar_wait(&S.vempty[s], ph, abort, status)) break;
                mbar_expect_tx(&S.vfull[s], kTileBytes);
                tma_load_4d(S.v[s], &tmV, &S.vfull[s], 0, kvh, k0, b);
                tma_load_4d(S.v[s] + kTileBytes / 2, &tmV, &S.vfull[s], 64, kvh, k0, b);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && nt > 0) {
            const uint32_t idS = idesc_bf16(128, 128, false, false);
            const uint32_t idPV = idesc_bf16(128, 128, false, true);
            const uint32_t qa = smem_u32(S.q);
            bool ok = mbar_wait(&S.bar_q, 0, abort, status);
            auto issue_s = [&](int n) -> bool {
                const int s = n & 1;
                if (!mbar_wait(&S.kfull[s], (n >> 1) & 1, abort, status)) return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(S.k[s]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
                    mma_ss(tmem + s * 128, sw128_desc(qa + off, 16, 1024),
                           sw128_desc(ka + off, 16, 1024), idS, kk > 0);
                }
                mma_commit(&S.kempty[s]);
                mma_commit(&S.sfull[s]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int n = 0; ok && n < nt; ++n) {
                const int s = n & 1;
                if (n + 1 < nt && !issue_s(n + 1)) break;
                if (!mbar_wait(&S.pfull[s], (n >> 1) & 1, abort, status)) break;
                if (!mbar_wait(&S.vfull[s], (n >> 1) & 1, abort, status)) break;
                tc_fence_after();
                const uint32_t va = smem_u32(S.v[s]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + 256, tmem + s * 128 + kk * 8,
                           sw128_desc(va + kk * 2048, kTileBytes / 2, 1024), idPV,
                           (n > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&S.vempty[s]);
                mma_commit(&S.odone);
            }
            // all issued MMAs complete before TMEM can be released
            mma_commit(&S.fin);
            wait_final(&S.fin, 0);
        }
    } else {
        // softmax warps: quadrant = warp % 4 selects TMEM lanes
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int t = q0 + row;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int n = 0; n < nt; ++n) {
            const int s = n & 1;
            const int32_t pid = m.row_pidx[e0 + n];
            uint4 bits = make_uint4(~0u, ~0u, ~0u, ~0u);
            if (pid >= 0)
                bits = *reinterpret_cast<const uint4 *>(m.bits + (int64_t)pid * 512 + row * 4);
            if (!__all_sync(0xffffffffu, mbar_wait(&S.sfull[s], (n >> 1) & 1, abort, status))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + s * 128 + c * 32, r[c]);
            tmem_ld_wait();
            const uint32_t wb[4] = {bits.x, bits.y, bits.z, bits.w};
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float x = __uint_as_float(r[c][j]) * scale_log2;
                    x = ((wb[c] >> j) & 1u) ? x : -INFINITY;
                    r[c][j] = __float_as_uint(x);
                    mt = fmaxf(mt, x);
                }
            const float m_new = fmaxf(m_run, mt);
            float alpha = 1.f;
            bool rescale = false;
            if (m_run == -INFINITY) {
                m_run = m_new;
            } else if (m_new > m_run + kRescaleThreshold) {
                alpha = ex2(m_run - m_new);
                m_run = m_new;
                l_run *= alpha;
                rescale = true;
            }
            if (__any_sync(0xffffffffu, rescale) && n > 0) {
                if (!__all_sync(0xffffffffu, mbar_wait(&S.odone, (n - 1) & 1, abort, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + 256 + c * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                    tmem_st32(tmem + lane_off + 256 + c * 32, o);
                }
            }
            const float mref = m_run == -INFINITY ? 0.f : m_run;
            float lsum = 0.f;
            uint32_t pk[2][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float p0 = ex2(__uint_as_float(r[c][j]) - mref);
                    const float p1 = ex2(__uint_as_float(r[c][j + 1]) - mref);
                    lsum += p0 + p1;
                    pk[c >> 1][(c & 1) * 16 + (j >> 1)] = pack_bf16(p0, p1);
                }
            l_run += lsum;
            tmem_st32(tmem + lane_off + s * 128, pk[0]);
            tmem_st32(tmem + lane_off + s * 128 + 32, pk[1]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&S.pfull[s]);
        }
        if (ok && nt > 0 &&
            __all_sync(0xffffffffu, mbar_wait(&S.odone, (nt - 1) & 1, abort, status))) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16 *orow = out + (((int64_t)b * N + t) * Hq + hq) * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + 256 + c * 32, o);
                tmem_ld_wait();
                if (t < N) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[j + 2]) * inv, __uint_as_float(o[j + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[j + 4]) * inv, __uint_as_float(o[j + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[j + 6]) * inv, __uint_as_float(o[j + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + j) = w;
                    }
                }
            }
            if (t < N)
                lse[((int64_t)b * Hq + hq) * N + t] =
                    l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B][N][H][128] bf16 viewed as 4-D (d, H, N, B); box = 64 x 1 x 128 x 1, 128-B swizzle.
bool make_tmap_bnhd(CUtensorMap *map, const void *base, int B, int N, int H) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {128 * 2, (cuuint64_t)H * 256, (cuuint64_t)N * H * 256};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_fwd_tc(const void *q, const void *k, const void *v, const kvs_tile_mask &m,
                          int32_t Hq, int32_t Hkv, float scale, void *o, float *lse,
                          int32_t *status, cudaStream_t s, bool *map_ok) {
    CUtensorMap tq, tk, tv;
    *map_ok = make_tmap_bnhd(&tq, q, m.B, m.N, Hq) && make_tmap_bnhd(&tk, k, m.B, m.N, Hkv) &&
              make_tmap_bnhd(&tv, v, m.B, m.N, Hkv);
    if (!*map_ok) return cudaSuccess;
    const size_t smem = sizeof(FwdSmem) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(k_attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (int64_t)m.B * Hq * m.T;
    k_attn_fwd_tc<<<(unsigned)grid, kFwdThreads, smem, s>>>(tq, tk, tv, m, Hq, Hkv,
                                                            scale * 1.4426950408889634f,
                                                            (__nv_bfloat16 *)o, lse, status);
    return cudaGetLastError();
}

}  // namespace kvs
