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
//   warp 1      TMEM allocator and tcgen05.mma issue (the whole warp runs the
//               loop, one lane chosen by elect.sync issues)
//   warps 2..5  softmax: thread = TMEM lane = query row
// TMEM (512 columns): S double buffer [0,128) [128,256), O accumulator [256,384).
// Per tile n: S_n = Q K_n^T (SS MMA) -> softmax reads S_n, writes P_n as bf16
// into the first 64 columns of the same buffer -> O += P_n V_n (A operand from
// TMEM). S_{n+1} is issued before PV_n, so the tensor core works on the next
// scores while the softmax warps handle the current ones. The running max is
// only raised (and O rescaled in TMEM) when it grows by more than 2^8;
// otherwise the stale max stays exact because O and the row sum share it.
#include <stdlib.h>

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
                  __nv_bfloat16 *__restrict__ out_lo, float *__restrict__ lse, int32_t *status) {
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
        if (nt > 0) {
            const bool leader = elect_one();
            const uint32_t idS = idesc_bf16(128, 128, false, false);
            const uint32_t idPV = idesc_bf16(128, 128, false, true);
            const uint64_t qd = sw128_desc(smem_u32(S.q), 16, 1024);
            const uint64_t kd0 = sw128_desc(smem_u32(S.k[0]), 16, 1024);
            const uint64_t kd1 = sw128_desc(smem_u32(S.k[1]), 16, 1024);
            const uint64_t vd0 = sw128_desc(smem_u32(S.v[0]), kTileBytes / 2, 1024);
            const uint64_t vd1 = sw128_desc(smem_u32(S.v[1]), kTileBytes / 2, 1024);
            bool ok = warp_wait(&S.bar_q, 0, abort, status);
            auto issue_s = [&](int n) -> bool {
                const int s = n & 1;
                if (!warp_wait(&S.kfull[s], (n >> 1) & 1, abort, status)) return false;
                tc_fence_after();
                const uint64_t kd = s ? kd1 : kd0;
                const uint32_t d = tmem + s * 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
                    if (leader) mma_ss(d, desc_add(qd, off), desc_add(kd, off), idS, kk > 0);
                }
                if (leader) mma_commit(&S.kempty[s]);
                if (leader) mma_commit(&S.sfull[s]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int n = 0; ok && n < nt; ++n) {
                const int s = n & 1;
                if (n + 1 < nt && !issue_s(n + 1)) break;
                if (!warp_wait(&S.pfull[s], (n >> 1) & 1, abort, status)) break;
                if (!warp_wait(&S.vfull[s], (n >> 1) & 1, abort, status)) break;
                tc_fence_after();
                const uint64_t vd = s ? vd1 : vd0;
                const uint32_t pa = tmem + s * 128, acc = n > 0 ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    if (leader) mma_ts(tmem + 256, pa + kk * 8, desc_add(vd, kk * 2048), idPV, kk > 0 ? 1u : acc);
                if (leader) mma_commit(&S.vempty[s]);
                if (leader) mma_commit(&S.odone);
            }
            // all issued MMAs complete before TMEM can be released
            if (leader) mma_commit(&S.fin);
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
            const int64_t orow = (((int64_t)b * N + t) * Hq + hq) * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + 256 + c * 32, o);
                tmem_ld_wait();
                if (t < N) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float x0 = __uint_as_float(o[j + 2 * u]) * inv;
                            const float x1 = __uint_as_float(o[j + 2 * u + 1]) * inv;
                            hi[u] = pack_bf16(x0, x1);
                            lo[u] = pack_bf16(x0 - bf16_lo(hi[u]), x1 - bf16_hi(hi[u]));
                        }
                        *reinterpret_cast<uint4 *>(out + orow + c * 32 + j) =
                            make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        if (out_lo)
                            *reinterpret_cast<uint4 *>(out_lo + orow + c * 32 + j) =
                                make_uint4(lo[0], lo[1], lo[2], lo[3]);
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

// ------------------------------------------------------------------ two heads per CTA
//
// Used when the group size G is even: the CTA takes query heads h0 and h0+1 of
// one kv group for the same query tile. Both heads share the tile list (the
// mask does not depend on the head) and every K/V tile, so each K/V tile is
// brought into shared memory once for two Q tiles. Two softmax warpgroups
// (warps 2..5 for h0, 6..9 for h0+1) alternate with the tensor core, which is
// fed in the order S0_n, S1_n, PV0_n, S0_{n+1}, PV1_n, S1_{n+1}, ...
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).

constexpr int kFwd2Threads = 320;

struct Fwd2Smem {
    uint8_t q[2][kTileBytes];
    uint8_t k[2][kTileBytes];
    uint8_t v[2][kTileBytes];
    // mask rows of tile n (partial tiles) in stage n % 4, loaded with K(n); stage
    // n % 4 is refilled only after K(n+2)'s stage was released, i.e. after both
    // softmax groups finished tile n+1 and so tile n
    uint32_t bits[4][128 * 4];
    int32_t pid[4];             // partial index of the tile in each bit stage (-1: full)
    uint64_t bar_q, kfull[2], kempty[2], vfull[2], vempty[2], sfull[2], pfull[2], odone[2], bfull[4], fin;
    uint32_t tmem_base;
    int abort;
};

__global__ void __launch_bounds__(kFwd2Threads, 1)
    k_attn_fwd_tc2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, kvs_tile_mask m, int32_t Hq,
                   int32_t Hkv, float scale_log2, __nv_bfloat16 *__restrict__ out,
                   __nv_bfloat16 *__restrict__ out_lo, float *__restrict__ lse, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    Fwd2Smem &S = *reinterpret_cast<Fwd2Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = m.B, N = m.N, T = m.T, G = Hq / Hkv, HP = Hq / 2;
    const int64_t idx = blockIdx.x;
    const int qi = T - 1 - (int)(idx / ((int64_t)B * HP));
    const int rem = (int)(idx % ((int64_t)B * HP));
    const int h0 = 2 * (rem % HP), b = rem / HP, kvh = h0 / G;
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
            mbar_init(&S.odone[i], 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&S.bfull[i], 1);
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
            mbar_expect_tx(&S.bar_q, 2 * kTileBytes);
            for (int x = 0; x < 2; ++x) {
                tma_load_4d(S.q[x], &tmQ, &S.bar_q, 0, h0 + x, q0, b);
                tma_load_4d(S.q[x] + kTileBytes / 2, &tmQ, &S.bar_q, 64, h0 + x, q0, b);
            }
            for (int n = 0; n < nt; ++n) {
                const int s = n & 1;
                const uint32_t ph = ((n >> 1) - 1) & 1;
                const int k0 = m.row_col[e0 + n] * 128;
                if (n >= 2 && !mbar_wait(&S.kempty[s], ph, abort, status)) break;
                mbar_expect_tx(&S.kfull[s], kTileBytes);
                tma_load_4d(S.k[s], &tmK, &S.kfull[s], 0, kvh, k0, b);
                tma_load_4d(S.k[s] + kTileBytes / 2, &tmK, &S.kfull[s], 64, kvh, k0, b);
                // the tile's mask rows go out with K, on their own 4-stage barrier, so
                // the softmax of tile n never waits for V(n)
                const int bsg = n & 3;
                const int32_t pid = m.row_pidx[e0 + n];
                S.pid[bsg] = pid;
                if (pid >= 0) {
                    mbar_expect_tx(&S.bfull[bsg], 2048u);
                    bulk_load(S.bits[bsg], m.bits + (int64_t)pid * 512, 2048, &S.bfull[bsg]);
                } else {
                    mbar_arrive(&S.bfull[bsg]);
                }
                if (n >= 2 && !mbar_wait(&S.vempty[s], ph, abort, status)) break;
                mbar_expect_tx(&S.vfull[s], kTileBytes);
                tma_load_4d(S.v[s], &tmV, &S.vfull[s], 0, kvh, k0, b);
                tma_load_4d(S.v[s] + kTileBytes / 2, &tmV, &S.vfull[s], 64, kvh, k0, b);
            }
        }
    } else if (warp == 1) {
        if (nt > 0) {
            const bool leader = elect_one();
            const uint32_t idS = idesc_bf16(128, 128, false, false);
            const uint32_t idPV = idesc_bf16(128, 128, false, true);
            const uint64_t qd0 = sw128_desc(smem_u32(S.q[0]), 16, 1024);
            const uint64_t qd1 = sw128_desc(smem_u32(S.q[1]), 16, 1024);
            const uint64_t kd0 = sw128_desc(smem_u32(S.k[0]), 16, 1024);
            const uint64_t kd1 = sw128_desc(smem_u32(S.k[1]), 16, 1024);
            const uint64_t vd0 = sw128_desc(smem_u32(S.v[0]), kTileBytes / 2, 1024);
            const uint64_t vd1 = sw128_desc(smem_u32(S.v[1]), kTileBytes / 2, 1024);
            auto issue_s = [&](int x, int n) {
                const uint64_t qd = x ? qd1 : qd0, kd = (n & 1) ? kd1 : kd0;
                const uint32_t d = tmem + x * 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
                    if (leader) mma_ss(d, desc_add(qd, off), desc_add(kd, off), idS, kk > 0);
                }
                if (leader) mma_commit(&S.sfull[x]);
            };
            auto issue_pv = [&](int x, int n) {
                const uint64_t vd = (n & 1) ? vd1 : vd0;
                const uint32_t d = tmem + 256 + x * 128, pa = tmem + x * 128, acc = n > 0 ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    if (leader) mma_ts(d, pa + kk * 8, desc_add(vd, kk * 2048), idPV, kk > 0 ? 1u : acc);
                if (leader) mma_commit(&S.odone[x]);
            };
            bool ok = warp_wait(&S.bar_q, 0, abort, status) &&
                      warp_wait(&S.kfull[0], 0, abort, status);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
                if (leader) mma_commit(&S.kempty[0]);
            }
            for (int n = 0; ok && n < nt; ++n) {
                const int s = n & 1;
                const bool more = n + 1 < nt;
                if (!warp_wait(&S.pfull[0], n & 1, abort, status)) break;
                if (!warp_wait(&S.vfull[s], (n >> 1) & 1, abort, status)) break;
                tc_fence_after();
                issue_pv(0, n);
                if (more) {
                    if (!warp_wait(&S.kfull[(n + 1) & 1], ((n + 1) >> 1) & 1, abort, status)) break;
                    tc_fence_after();
                    issue_s(0, n + 1);
                }
                if (!warp_wait(&S.pfull[1], n & 1, abort, status)) break;
                tc_fence_after();
                issue_pv(1, n);
                if (leader) mma_commit(&S.vempty[s]);
                if (more) {
                    issue_s(1, n + 1);
                    if (leader) mma_commit(&S.kempty[(n + 1) & 1]);
                }
            }
            if (leader) mma_commit(&S.fin);
            wait_final(&S.fin, 0);
        }
    } else {
        const int x = (warp - 2) >> 2;           // which head of the pair
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int t = q0 + row;
        const int hq = h0 + x;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t cS = x * 128, cO = 256 + x * 128;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int n = 0; n < nt; ++n) {
            if (!__all_sync(0xffffffffu, mbar_wait(&S.sfull[x], n & 1, abort, status))) {
                ok = false;
                break;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&S.bfull[n & 3], (n >> 2) & 1, abort, status))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool partial = S.pid[n & 3] >= 0;  // same for the whole CTA
            uint4 bits = make_uint4(~0u, ~0u, ~0u, ~0u);
            if (partial) bits = *reinterpret_cast<const uint4 *>(&S.bits[n & 3][row * 4]);
            const uint32_t wb[4] = {bits.x, bits.y, bits.z, bits.w};
            // pass 1: row maximum of the (masked) raw scores; 8 independent partial
            // maxima keep the reduction off one serial dependency chain
            float mx8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_off + cS + hc * 64, r0);
                tmem_ld32(tmem + lane_off + cS + hc * 64 + 32, r1);
                tmem_ld_wait();
                if (partial) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if ((wb[2 * hc] >> j) & 1u) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(r0[j]));
                        if ((wb[2 * hc + 1] >> j) & 1u) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(r1[j]));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        mx8[j & 7] = max3f(mx8[j & 7], __uint_as_float(r0[j]), __uint_as_float(r1[j]));
                }
            }
            float mraw = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float mt = mraw * scale_log2;  // scale_log2 > 0 keeps the order
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
                if (!__all_sync(0xffffffffu, mbar_wait(&S.odone[x], (n - 1) & 1, abort, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + cO + c * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                    tmem_st32(tmem + lane_off + cO + c * 32, o);
                }
            }
            // pass 2: P = 2^(s*c - m) as bf16 pairs over the first 64 columns of S
            // (the two 32-column chunks of a half are read before their 32 packed
            // columns overwrite the first of them). Half of the exponentials run on
            // the FMA pipe (exp2_fma), half on the special-function unit.
            const float nref = m_run == -INFINITY ? 0.f : -m_run;
            uint64_t lsum2[4];  // four f32x2 partial row sums
#pragma unroll
            for (int u = 0; u < 4; ++u) lsum2[u] = 0ull;
#pragma unroll 1
            for (int hc = 0; hc < 2; ++hc) {
                uint32_t r0[32], r1[32], pk[32];
                tmem_ld32(tmem + lane_off + cS + hc * 64, r0);
                tmem_ld32(tmem + lane_off + cS + hc * 64 + 32, r1);
                tmem_ld_wait();
                const uint32_t w0 = hc ? wb[2] : wb[0], w1 = hc ? wb[3] : wb[1];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t(&r)[32] = cc ? r1 : r0;
                    const uint32_t w = cc ? w1 : w0;
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float x0, x1, x2, x3, p0, p1;
                        fma2(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), scale_log2, nref, x0, x1);
                        fma2(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]), scale_log2, nref, x2, x3);
                        exp2_fma_x2(x0, x1, p0, p1);
                        float p2 = ex2(x2), p3 = ex2(x3);
                        if (partial) {
                            p0 = ((w >> j) & 1u) ? p0 : 0.f;
                            p1 = ((w >> (j + 1)) & 1u) ? p1 : 0.f;
                            p2 = ((w >> (j + 2)) & 1u) ? p2 : 0.f;
                            p3 = ((w >> (j + 3)) & 1u) ? p3 : 0.f;
                        }
                        const int a = ((j >> 2) & 1) * 2;
                        lsum2[a] = f2_add(lsum2[a], f2_make(p0, p1));
                        lsum2[a + 1] = f2_add(lsum2[a + 1], f2_make(p2, p3));
                        pk[cc * 16 + (j >> 1)] = pack_bf16(p0, p1);
                        pk[cc * 16 + (j >> 1) + 1] = pack_bf16(p2, p3);
                    }
                }
                tmem_st32(tmem + lane_off + cS + hc * 32, pk);
            }
            float ls[8];
            f2_split(f2_add(lsum2[0], lsum2[2]), ls[0], ls[1]);
            f2_split(f2_add(lsum2[1], lsum2[3]), ls[2], ls[3]);
            l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&S.pfull[x]);
        }
        if (ok && nt > 0 &&
            __all_sync(0xffffffffu, mbar_wait(&S.odone[x], (nt - 1) & 1, abort, status))) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            const int64_t orow = (((int64_t)b * N + t) * Hq + hq) * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + cO + c * 32, o);
                tmem_ld_wait();
                if (t < N) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float x0 = __uint_as_float(o[j + 2 * u]) * inv;
                            const float x1 = __uint_as_float(o[j + 2 * u + 1]) * inv;
                            hi[u] = pack_bf16(x0, x1);
                            lo[u] = pack_bf16(x0 - bf16_lo(hi[u]), x1 - bf16_hi(hi[u]));
                        }
                        *reinterpret_cast<uint4 *>(out + orow + c * 32 + j) =
                            make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        if (out_lo)
                            *reinterpret_cast<uint4 *>(out_lo + orow + c * 32 + j) =
                                make_uint4(lo[0], lo[1], lo[2], lo[3]);
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

// ------------------------------------------------------------------ two heads, one pass over S
//
// The same schedule as k_attn_fwd_tc2 with the softmax reading each S tile in
// one pass: all 128 score columns of a row come into registers with a single
// TMEM round trip (about 194 registers per softmax thread). P is handed to the
// MMA warp in two halves of 64 keys: PV's first four k-steps run while the
// softmax still computes the second half, which shortens each head's
// S -> softmax -> PV -> next S chain. The block has three
// warpgroups of 128 threads -- warp 0 TMA, warp 1 MMA, warps 2-3 idle; warps
// 4-7 head h0; warps 8-11 head h0+1 -- launched at 168 registers per thread;
// after set-up the first warpgroup gives registers back (setmaxnreg.dec to 88)
// and the softmax warpgroups take them (setmaxnreg.inc to 208):
// 88 + 208 + 208 = 3 x 168, exactly the block's launch allocation. The host
// launches this kernel only when the compiled kernel uses exactly 168
// registers per thread, so the split always adds up.
constexpr int kFwd3Threads = 384;
constexpr int kFwd3Regs = 168, kFwd3RegsLow = 88, kFwd3RegsHigh = 208;
static_assert(kFwd3RegsLow + 2 * kFwd3RegsHigh == 3 * kFwd3Regs, "register split must equal the launch allocation");

struct Fwd3Smem {  // as Fwd2Smem, plus the skip flag
    uint8_t q[2][kTileBytes];
    uint8_t k[2][kTileBytes];
    uint8_t v[2][kTileBytes];
    // mask rows of tile n (partial tiles) in stage n % 4, loaded with K(n); stage
    // n % 4 is refilled only after K(n+2)'s stage was released, i.e. after both
    // softmax groups finished tile n+1 and so tile n
    uint32_t bits[4][128 * 4];
    int32_t pid[4];             // partial index of the tile in each bit stage (-1: full)
    // pfull[x][hc]: head x's P for keys 64hc..64hc+63 is in TMEM
    uint64_t bar_q, kfull[2], kempty[2], vfull[2], vempty[2], sfull[2], pfull[2][2], odone[2], bfull[4], fin;
    uint32_t tmem_base;
    int abort;
    int skip;
};

__global__ void __launch_bounds__(kFwd3Threads, 1)
    k_attn_fwd_tc3(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, kvs_tile_mask m, int32_t Hq,
                   int32_t Hkv, float scale_log2, __nv_bfloat16 *__restrict__ out,
                   __nv_bfloat16 *__restrict__ out_lo, float *__restrict__ lse, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    Fwd3Smem &S = *reinterpret_cast<Fwd3Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = m.B, N = m.N, T = m.T, G = Hq / Hkv, HP = Hq / 2;
    const int64_t idx = blockIdx.x;
    const int qi = T - 1 - (int)(idx / ((int64_t)B * HP));
    const int rem = (int)(idx % ((int64_t)B * HP));
    const int h0 = 2 * (rem % HP), b = rem / HP, kvh = h0 / G;
    const int q0 = qi * 128;
    const int32_t e0 = m.row_ptr[b * T + qi], nt_list = m.row_ptr[b * T + qi + 1] - e0;
    // every thread must reach setmaxnreg below: a CTA that finds the grid timed out
    // skips its work (nt = 0) instead of returning, decided once by thread 0

    if (threadIdx.x == 0) {
        S.skip = grid_timed_out(status) ? 1 : 0;
        mbar_init(&S.bar_q, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.kfull[i], 1);
            mbar_init(&S.kempty[i], 1);
            mbar_init(&S.vfull[i], 1);
            mbar_init(&S.vempty[i], 1);
            mbar_init(&S.sfull[i], 1);
            mbar_init(&S.pfull[i][0], 128);
            mbar_init(&S.pfull[i][1], 128);
            mbar_init(&S.odone[i], 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&S.bfull[i], 1);
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
    const int32_t nt = S.skip ? 0 : nt_list;
    if (warp < 4) {
        // first warpgroup: TMA (warp 0) and MMA (warp 1) need few registers
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kFwd3RegsLow));
        if (warp == 0) {
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_expect_tx(&S.bar_q, 2 * kTileBytes);
            for (int x = 0; x < 2; ++x) {
                tma_load_4d(S.q[x], &tmQ, &S.bar_q, 0, h0 + x, q0, b);
                tma_load_4d(S.q[x] + kTileBytes / 2, &tmQ, &S.bar_q, 64, h0 + x, q0, b);
            }
            for (int n = 0; n < nt; ++n) {
                const int s = n & 1;
                const uint32_t ph = ((n >> 1) - 1) & 1;
                const int k0 = m.row_col[e0 + n] * 128;
                if (n >= 2 && !mbar_wait(&S.kempty[s], ph, abort, status)) break;
                mbar_expect_tx(&S.kfull[s], kTileBytes);
                tma_load_4d(S.k[s], &tmK, &S.kfull[s], 0, kvh, k0, b);
                tma_load_4d(S.k[s] + kTileBytes / 2, &tmK, &S.kfull[s], 64, kvh, k0, b);
                // the tile's mask rows go out with K, on their own 4-stage barrier, so
                // the softmax of tile n never waits for V(n)
                const int bsg = n & 3;
                const int32_t pid = m.row_pidx[e0 + n];
                S.pid[bsg] = pid;
                if (pid >= 0) {
                    mbar_expect_tx(&S.bfull[bsg], 2048u);
                    bulk_load(S.bits[bsg], m.bits + (int64_t)pid * 512, 2048, &S.bfull[bsg]);
                } else {
                    mbar_arrive(&S.bfull[bsg]);
                }
                if (n >= 2 && !mbar_wait(&S.vempty[s], ph, abort, status)) break;
                mbar_expect_tx(&S.vfull[s], kTileBytes);
                tma_load_4d(S.v[s], &tmV, &S.vfull[s], 0, kvh, k0, b);
                tma_load_4d(S.v[s] + kTileBytes / 2, &tmV, &S.vfull[s], 64, kvh, k0, b);
            }
        }
    } else if (warp == 1) {
        if (nt > 0) {
            const bool leader = elect_one();
            const uint32_t idS = idesc_bf16(128, 128, false, false);
            const uint32_t idPV = idesc_bf16(128, 128, false, true);
            const uint64_t qd0 = sw128_desc(smem_u32(S.q[0]), 16, 1024);
            const uint64_t qd1 = sw128_desc(smem_u32(S.q[1]), 16, 1024);
            const uint64_t kd0 = sw128_desc(smem_u32(S.k[0]), 16, 1024);
            const uint64_t kd1 = sw128_desc(smem_u32(S.k[1]), 16, 1024);
            const uint64_t vd0 = sw128_desc(smem_u32(S.v[0]), kTileBytes / 2, 1024);
            const uint64_t vd1 = sw128_desc(smem_u32(S.v[1]), kTileBytes / 2, 1024);
            auto issue_s = [&](int x, int n) {
                const uint64_t qd = x ? qd1 : qd0, kd = (n & 1) ? kd1 : kd0;
                const uint32_t d = tmem + x * 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
                    if (leader) mma_ss(d, desc_add(qd, off), desc_add(kd, off), idS, kk > 0);
                }
                if (leader) mma_commit(&S.sfull[x]);
            };
            // PV(n) of head x in two halves of 64 keys, each issued once the softmax
            // has written that half of P
            auto issue_pv = [&](int x, int n) -> bool {
                const uint64_t vd = (n & 1) ? vd1 : vd0;
                const uint32_t d = tmem + 256 + x * 128, pa = tmem + x * 128, acc = n > 0 ? 1u : 0u;
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    if (!warp_wait(&S.pfull[x][hc], n & 1, abort, status)) return false;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 4 * hc; kk < 4 * hc + 4; ++kk)
                        if (leader) mma_ts(d, pa + kk * 8, desc_add(vd, kk * 2048), idPV, kk > 0 ? 1u : acc);
                }
                if (leader) mma_commit(&S.odone[x]);
                return true;
            };
            bool ok = warp_wait(&S.bar_q, 0, abort, status) &&
                      warp_wait(&S.kfull[0], 0, abort, status);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
                if (leader) mma_commit(&S.kempty[0]);
            }
            for (int n = 0; ok && n < nt; ++n) {
                const int s = n & 1;
                const bool more = n + 1 < nt;
                if (!warp_wait(&S.vfull[s], (n >> 1) & 1, abort, status)) break;
                if (!issue_pv(0, n)) break;
                if (more) {
                    if (!warp_wait(&S.kfull[(n + 1) & 1], ((n + 1) >> 1) & 1, abort, status)) break;
                    tc_fence_after();
                    issue_s(0, n + 1);
                }
                if (!issue_pv(1, n)) break;
                if (leader) mma_commit(&S.vempty[s]);
                if (more) {
                    issue_s(1, n + 1);
                    if (leader) mma_commit(&S.kempty[(n + 1) & 1]);
                }
            }
            if (leader) mma_commit(&S.fin);
            wait_final(&S.fin, 0);
        }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kFwd3RegsHigh));
        const int x = (warp - 4) >> 2;           // which head of the pair
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const int t = q0 + row;
        const int hq = h0 + x;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t cS = x * 128, cO = 256 + x * 128;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int n = 0; n < nt; ++n) {
            if (!__all_sync(0xffffffffu, mbar_wait(&S.sfull[x], n & 1, abort, status))) {
                ok = false;
                break;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&S.bfull[n & 3], (n >> 2) & 1, abort, status))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool partial = S.pid[n & 3] >= 0;  // same for the whole CTA
            uint4 bits = make_uint4(~0u, ~0u, ~0u, ~0u);
            if (partial) bits = *reinterpret_cast<const uint4 *>(&S.bits[n & 3][row * 4]);
            const uint32_t wb[4] = {bits.x, bits.y, bits.z, bits.w};
            // one pass over S: all 128 columns of this row come into registers with one
            // TMEM round trip; 8 independent partial maxima keep the reduction off one
            // serial dependency chain
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + cS + c * 32, r[c]);
            tmem_ld_wait();
            float mx8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
            if (partial) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if ((wb[c] >> j) & 1u) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(r[c][j]));
            } else {
#pragma unroll
                for (int c = 0; c < 4; c += 2)
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        mx8[j & 7] = max3f(mx8[j & 7], __uint_as_float(r[c][j]), __uint_as_float(r[c + 1][j]));
            }
            float mraw = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float mt = mraw * scale_log2;  // scale_log2 > 0 keeps the order
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
                if (!__all_sync(0xffffffffu, mbar_wait(&S.odone[x], (n - 1) & 1, abort, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + cO + c * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                    tmem_st32(tmem + lane_off + cO + c * 32, o);
                }
            }
            // P = 2^(s*c - m) as bf16 pairs into the first 64 columns of S (all of S is
            // already in registers), all exponentials on the special-function unit: with P
            // handed over in halves this kernel is bound by the softmax's instruction
            // latency, and ex2.approx is one instruction per value where the FMA-pipe
            // cubic takes about five.
            const float nref = m_run == -INFINITY ? 0.f : -m_run;
            uint64_t lsum2[4];  // four f32x2 partial row sums
#pragma unroll
            for (int u = 0; u < 4; ++u) lsum2[u] = 0ull;
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
                uint32_t pk[32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t(&rr)[32] = r[2 * hc + cc];
                    const uint32_t w = wb[2 * hc + cc];
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float x0, x1, x2, x3, p0, p1;
                        fma2(__uint_as_float(rr[j]), __uint_as_float(rr[j + 1]), scale_log2, nref, x0, x1);
                        fma2(__uint_as_float(rr[j + 2]), __uint_as_float(rr[j + 3]), scale_log2, nref, x2, x3);
                        p0 = ex2(x0);
                        p1 = ex2(x1);
                        float p2 = ex2(x2), p3 = ex2(x3);
                        if (partial) {
                            p0 = ((w >> j) & 1u) ? p0 : 0.f;
                            p1 = ((w >> (j + 1)) & 1u) ? p1 : 0.f;
                            p2 = ((w >> (j + 2)) & 1u) ? p2 : 0.f;
                            p3 = ((w >> (j + 3)) & 1u) ? p3 : 0.f;
                        }
                        const int a = ((j >> 2) & 1) * 2;
                        lsum2[a] = f2_add(lsum2[a], f2_make(p0, p1));
                        lsum2[a + 1] = f2_add(lsum2[a + 1], f2_make(p2, p3));
                        pk[cc * 16 + (j >> 1)] = pack_bf16(p0, p1);
                        pk[cc * 16 + (j >> 1) + 1] = pack_bf16(p2, p3);
                    }
                }
                tmem_st32(tmem + lane_off + cS + hc * 32, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&S.pfull[x][hc]);  // this half of P is ready for PV
            }
            float ls[8];
            f2_split(f2_add(lsum2[0], lsum2[2]), ls[0], ls[1]);
            f2_split(f2_add(lsum2[1], lsum2[3]), ls[2], ls[3]);
            l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        }
        if (ok && nt > 0 &&
            __all_sync(0xffffffffu, mbar_wait(&S.odone[x], (nt - 1) & 1, abort, status))) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            const int64_t orow = (((int64_t)b * N + t) * Hq + hq) * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + cO + c * 32, o);
                tmem_ld_wait();
                if (t < N) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float x0 = __uint_as_float(o[j + 2 * u]) * inv;
                            const float x1 = __uint_as_float(o[j + 2 * u + 1]) * inv;
                            hi[u] = pack_bf16(x0, x1);
                            lo[u] = pack_bf16(x0 - bf16_lo(hi[u]), x1 - bf16_hi(hi[u]));
                        }
                        *reinterpret_cast<uint4 *>(out + orow + c * 32 + j) =
                            make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        if (out_lo)
                            *reinterpret_cast<uint4 *>(out_lo + orow + c * 32 + j) =
                                make_uint4(lo[0], lo[1], lo[2], lo[3]);
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
// [B, N, H, 128] bf16, boxes of 64 dims x box_rows tokens of one head, 128-byte swizzle.
bool make_tmap_bnhd(CUtensorMap *map, const void *base, int B, int N, int H, int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {128 * 2, (cuuint64_t)H * 256, (cuuint64_t)N * H * 256};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The one-pass kernel's register split (setmaxnreg) must add up to the block's
// launch allocation, which holds only when the compiled kernel uses exactly
// kFwd3Regs registers per thread; otherwise (or with KVS_FWD_ONEPASS=0 in the
// environment) the two-pass kernel runs.
static bool fwd_one_pass_ok() {
    static int ok = -1;
    if (ok < 0) {
        cudaFuncAttributes a;
        const char *env = getenv("KVS_FWD_ONEPASS");
        ok = (!env || env[0] != '0') && cudaFuncGetAttributes(&a, k_attn_fwd_tc3) == cudaSuccess &&
             a.numRegs == kFwd3Regs && a.maxThreadsPerBlock >= kFwd3Threads;
    }
    return ok == 1;
}

cudaError_t launch_fwd_tc(const void *q, const void *k, const void *v, const kvs_tile_mask &m,
                          int32_t Hq, int32_t Hkv, float scale, void *o, void *o_lo, float *lse,
                          int32_t *status, cudaStream_t s, bool *map_ok) {
    CUtensorMap tq, tk, tv;
    *map_ok = make_tmap_bnhd(&tq, q, m.B, m.N, Hq, 128) && make_tmap_bnhd(&tk, k, m.B, m.N, Hkv, 128) &&
              make_tmap_bnhd(&tv, v, m.B, m.N, Hkv, 128);
    if (!*map_ok) return cudaSuccess;
    const int G = Hq / Hkv;
    const float sl2 = scale * 1.4426950408889634f;
    if (G % 2 == 0 && fwd_one_pass_ok()) {
        const size_t smem = sizeof(Fwd3Smem) + 1024;
        cudaError_t e = cudaFuncSetAttribute(k_attn_fwd_tc3, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t grid = (int64_t)m.B * (Hq / 2) * m.T;
        k_attn_fwd_tc3<<<(unsigned)grid, kFwd3Threads, smem, s>>>(
            tq, tk, tv, m, Hq, Hkv, sl2, (__nv_bfloat16 *)o, (__nv_bfloat16 *)o_lo, lse, status);
    } else if (G % 2 == 0) {
        const size_t smem = sizeof(Fwd2Smem) + 1024;
        cudaError_t e = cudaFuncSetAttribute(k_attn_fwd_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t grid = (int64_t)m.B * (Hq / 2) * m.T;
        k_attn_fwd_tc2<<<(unsigned)grid, kFwd2Threads, smem, s>>>(
            tq, tk, tv, m, Hq, Hkv, sl2, (__nv_bfloat16 *)o, (__nv_bfloat16 *)o_lo, lse, status);
    } else {
        const size_t smem = sizeof(FwdSmem) + 1024;
        cudaError_t e = cudaFuncSetAttribute(k_attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t grid = (int64_t)m.B * Hq * m.T;
        k_attn_fwd_tc<<<(unsigned)grid, kFwdThreads, smem, s>>>(
            tq, tk, tv, m, Hq, Hkv, sl2, (__nv_bfloat16 *)o, (__nv_bfloat16 *)o_lo, lse, status);
    }
    return cudaGetLastError();
}

}  // namespace kvs
