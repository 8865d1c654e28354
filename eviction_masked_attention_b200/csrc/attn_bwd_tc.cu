// bf16 eviction-masked attention backward on sm_100a tensor cores.
//
// Textbook softmax-attention gradients restricted to the visible pairs of the
// replayed trace ("KV-streams: speeding up agentic RL by operating on the KV
// cache directly", trainer replay; "KV-streams for Efficient Compaction in
// Agentic Reinforcement Learning", Fig. 2(A)):
//   P = exp(S - LSE), dV = P^T dO, dP = dO V^T, dS = P (dP - D),
//   dQ = scale dS K, dK = scale dS^T Q, D = rowsum(dO * O).
//
// Three launches, no atomics (deterministic):
//   prep   D and -LSE*log2(e) per (trace, head, row), padded to whole tiles
//   dK/dV  one CTA per (key tile, kv head, trace); walks the column lists of
//          the mask for every query head of the group, one 128-row query tile
//          per item. Transposed products S^T = K Q^T and dP^T = V dO^T put one
//          key per TMEM lane, so P^T and dS^T are written back to TMEM in bf16
//          and used as the A operand of dV += P^T dO and dK += dS^T Q; the
//          next item's S^T and dP^T are issued between them so the elementwise
//          phases overlap tensor work. Within a tile a key's visible query rows
//          form one interval (j <= t < kappa_j), so masking needs only kappa_j,
//          not the bit rows.
//   dQ     one CTA per (query tile, head, trace) over the row lists:
//          S = Q K^T, dP = dO V^T, dS (bit-masked) to TMEM, dQ += dS K.
// Warp roles: warp 0 TMA, warp 1 TMEM + MMA issue (the whole warp runs the
// loop, one elected lane issues), warps 2..17 elementwise (thread = TMEM lane).
#include "common.cuh"

namespace kvs {

bool make_tmap_bnhd(CUtensorMap *map, const void *base, int B, int N, int H, int box_rows);

constexpr uint32_t kTile = 128 * 128 * 2;

__device__ __forceinline__ bool wait_done(uint64_t *bar, uint32_t parity) {
    uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}


// D[b][h][t] = <dO, O>, NL2[b][h][t] = -lse * log2(e) (so that the exponent of P is one
// fma of the raw score); rows t >= N get 0. Tpad = T*128.
// O is o_hi (+ o_lo when the forward kept the rounding residual of its output).
__global__ void k_bwd_prep(const __nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ o_lo,
                           const __nv_bfloat16 *__restrict__ dO, const float *__restrict__ lse,
                           int32_t B, int32_t N, int32_t Hq, int32_t Tpad, float *__restrict__ Drow,
                           float *__restrict__ NL2) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (int64_t)B * Hq * Tpad) return;
    const int64_t t = row % Tpad, bh = row / Tpad, h = bh % Hq, b = bh / Hq;
    float s = 0.f, nl2 = 0.f;
    if (t < N) {
        const int64_t off = ((b * N + t) * Hq + h) * 128 + lane * 4;
        const uint2 a = *reinterpret_cast<const uint2 *>(o + off);
        const uint2 c = *reinterpret_cast<const uint2 *>(dO + off);
        float o0 = bf16_lo(a.x), o1 = bf16_hi(a.x), o2 = bf16_lo(a.y), o3 = bf16_hi(a.y);
        if (o_lo) {
            const uint2 r = *reinterpret_cast<const uint2 *>(o_lo + off);
            o0 += bf16_lo(r.x); o1 += bf16_hi(r.x); o2 += bf16_lo(r.y); o3 += bf16_hi(r.y);
        }
        s = o0 * bf16_lo(c.x) + o1 * bf16_hi(c.x) + o2 * bf16_lo(c.y) + o3 * bf16_hi(c.y);
        for (int k = 16; k; k >>= 1) s += __shfl_xor_sync(0xffffffffu, s, k);
        nl2 = -lse[(b * Hq + h) * N + t] * 1.4426950408889634f;
    }
    if (lane == 0) {
        Drow[row] = s;
        NL2[row] = nl2;
    }
}

// Store 32 fp32 values (times f) of a row as bf16 to 64 contiguous bytes.
__device__ __forceinline__ void store_row32(__nv_bfloat16 *dst, const uint32_t (&r)[32], float f) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
        uint4 w;
        w.x = pack_bf16(__uint_as_float(r[j]) * f, __uint_as_float(r[j + 1]) * f);
        w.y = pack_bf16(__uint_as_float(r[j + 2]) * f, __uint_as_float(r[j + 3]) * f);
        w.z = pack_bf16(__uint_as_float(r[j + 4]) * f, __uint_as_float(r[j + 5]) * f);
        w.w = pack_bf16(__uint_as_float(r[j + 6]) * f, __uint_as_float(r[j + 7]) * f);
        *reinterpret_cast<uint4 *>(dst + j) = w;
    }
}


// ---------------------------------------------------------------------- dK / dV
//
// An item is (128-row query tile of the key tile's column list, query head of
// the group). TMEM: S^T [0,128) and dP^T [128,256) of the current item, dV
// [256,384), dK [384,512). Sixteen elementwise warps (four per TMEM lane
// quarter, so that each scheduler has four to hide the TMEM and exponential
// latencies) split an item's rows in four parts (part p takes rows
// 32p..32p+31, thread = key lane); each writes its P^T (dS^T) as bf16 pairs
// into the first 16 of its own 32 columns of S^T (dP^T), so no part overwrites
// scores another still reads. Per item the tensor core runs, in issue order,
//   dV(n) += P^T(n) dO(n), S^T(n+1) = K Q(n+1)^T, dK(n) += dS^T(n) Q(n),
//   dP^T(n+1) = V dO(n+1)^T
// (four M=128 N=128 K=128 products): the elementwise phase P^T(n+1) runs while
// dK(n) and dP^T(n+1) execute, and dS^T(n) while dV(n) and S^T(n+1) execute.
// P^T and dS^T reach the MMA warp in two halves (the first and second 16 rows
// of every 32-row part, k-steps 0, 2, 4, 6 and 1, 3, 5, 7 of dV or dK), so each
// product starts while the elementwise warps still compute its second half.
// Each product that overwrites a TMEM region is issued after the product that
// reads it (MMAs run in issue order) and after the elementwise warps reported
// they had read it.

constexpr int kBwdEwThreads = 512;               // 16 elementwise warps
constexpr int kBwdThreads = 64 + kBwdEwThreads;  // warp 0 TMA, warp 1 MMA, warps 2..17 elementwise
// Q(n) is read by S^T(n) and dK(n), dO(n) by dP^T(n) and dV(n). With three Q
// stages the load of Q(n+3) goes out when dK(n) completes, six products before
// S^T(n+3); with two dO stages the load of dO(n+2) goes out when dV(n)
// completes, six products before dP^T(n+2). The rows' -LSE log2(e) and D (and
// the tile's origin and class) ride on a 2-stage ring of their own that the
// elementwise warps release when they finish an item.
constexpr int kDkvQStages = 3, kDkvOStages = 2, kDkvRowStages = 2;

struct DkvSmem {
    uint8_t k[kTile];
    uint8_t v[kTile];
    uint8_t q[kDkvQStages][kTile];
    uint8_t dout[kDkvOStages][kTile];
    float nl2[kDkvRowStages][128];  // -lse log2(e) of the tile's rows
    float dd[kDkvRowStages][128];
    int32_t q0[kDkvRowStages], full_tile[kDkvRowStages];  // tile origin, FULL flag
    uint64_t kv_full, qfull[kDkvQStages], qempty[kDkvQStages], ofull[kDkvOStages], oempty[kDkvOStages],
        rfull[kDkvRowStages], rempty[kDkvRowStages], st_full, dp_full, p_ready[2], ds_ready[2], acc_done, fin;
    uint32_t tmem_base;
    int abort;
};
// the whole budget of dynamic shared memory; the kernel checks that its base is
// 1024-byte aligned (the swizzled tiles need it) instead of padding for it
static_assert(sizeof(DkvSmem) <= 232448, "dK/dV shared memory over the 227 KB limit");

// TMEM column of the bf16 pairs of rows (keys) 16kk..16kk+15 inside a 128-column
// region whose four 32-column parts hold rows 32p..32p+31 in their first 16 columns.
__device__ __forceinline__ uint32_t part_col(int kk) { return 32 * (kk >> 1) + 8 * (kk & 1); }

__global__ void __launch_bounds__(kBwdThreads, 1)
    k_attn_dkdv_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   kvs_tile_mask m, int32_t Hq, int32_t Hkv, float scale, float scale_log2,
                   const float *__restrict__ Drow, const float *__restrict__ NL2,
                   __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv, int32_t *status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    DkvSmem &S = *reinterpret_cast<DkvSmem *>(smem_raw);
    if (smem_u32(smem_raw) & 1023u) {  // same for every thread of the CTA
        if (threadIdx.x == 0) set_status(status, KVS_ERR_UNSUPPORTED);
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = m.B, N = m.N, T = m.T, G = Hq / Hkv, Tpad = T * 128;
    // key tiles with the longest column lists (small kj) first
    const int64_t idx = blockIdx.x;
    const int kj = (int)(idx / ((int64_t)B * Hkv));
    const int rem = (int)(idx % ((int64_t)B * Hkv));
    const int kvh = rem % Hkv, b = rem / Hkv;
    const int k0 = kj * 128;
    const int32_t c0 = m.col_ptr[b * T + kj], ncol = m.col_ptr[b * T + kj + 1] - c0;
    const int nw = ncol * G;
    if (grid_timed_out(status)) return;

    if (threadIdx.x == 0) {
        mbar_init(&S.kv_full, 1);
        for (int i = 0; i < kDkvQStages; ++i) {
            mbar_init(&S.qfull[i], 1);
            mbar_init(&S.qempty[i], 1);
        }
        for (int i = 0; i < kDkvOStages; ++i) {
            mbar_init(&S.ofull[i], 1);
            mbar_init(&S.oempty[i], 1);
        }
        for (int i = 0; i < kDkvRowStages; ++i) {
            mbar_init(&S.rfull[i], 1);
            mbar_init(&S.rempty[i], kBwdEwThreads);
        }
        mbar_init(&S.st_full, 1);
        mbar_init(&S.dp_full, 1);
        for (int i = 0; i < 2; ++i) {  // halves h: k-steps h, h+2, h+4, h+6 of dV / dK
            mbar_init(&S.p_ready[i], kBwdEwThreads);
            mbar_init(&S.ds_ready[i], kBwdEwThreads);
        }
        mbar_init(&S.acc_done, 1);
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
    constexpr uint32_t cST = 0, cDP = 128, cDV = 256, cDK = 384;

    if (warp == 0) {
        if (lane == 0 && nw > 0) {
            mbar_expect_tx(&S.kv_full, 2 * kTile);
            tma_load_4d(S.k, &tmK, &S.kv_full, 0, kvh, k0, b);
            tma_load_4d(S.k + kTile / 2, &tmK, &S.kv_full, 64, kvh, k0, b);
            tma_load_4d(S.v, &tmV, &S.kv_full, 0, kvh, k0, b);
            tma_load_4d(S.v + kTile / 2, &tmV, &S.kv_full, 64, kvh, k0, b);
            // Q(n) once dK(n-3) is done, dO(n) once dV(n-2) is done
            for (int n = 0; n < nw; ++n) {
                const int e = n / G, h = kvh * G + n % G;
                const int q0 = m.col_row[c0 + e] * 128;
                const int qs = n % kDkvQStages;
                if (n >= kDkvQStages &&
                    !mbar_wait(&S.qempty[qs], ((n / kDkvQStages) - 1) & 1, abort, status))
                    break;
                mbar_expect_tx(&S.qfull[qs], kTile);
                tma_load_4d(S.q[qs], &tmQ, &S.qfull[qs], 0, h, q0, b);
                tma_load_4d(S.q[qs] + kTile / 2, &tmQ, &S.qfull[qs], 64, h, q0, b);
                const int os = n % kDkvOStages;
                if (n >= kDkvOStages &&
                    !mbar_wait(&S.oempty[os], ((n / kDkvOStages) - 1) & 1, abort, status))
                    break;
                mbar_expect_tx(&S.ofull[os], kTile);
                tma_load_4d(S.dout[os], &tmO, &S.ofull[os], 0, h, q0, b);
                tma_load_4d(S.dout[os] + kTile / 2, &tmO, &S.ofull[os], 64, h, q0, b);
            }
        } else if (lane == 1 && nw > 0) {
            // the items' row data, each once the elementwise warps are done with item n-2
            for (int n = 0; n < nw; ++n) {
                const int e = n / G, h = kvh * G + n % G;
                const int q0 = m.col_row[c0 + e] * 128;
                const int64_t ro = ((int64_t)b * Hq + h) * Tpad + q0;
                const int rs = n % kDkvRowStages;
                if (n >= kDkvRowStages &&
                    !mbar_wait(&S.rempty[rs], ((n / kDkvRowStages) - 1) & 1, abort, status))
                    break;
                S.q0[rs] = q0;
                S.full_tile[rs] = m.col_pidx[c0 + e] < 0;
                mbar_expect_tx(&S.rfull[rs], 1024);
                bulk_load(S.nl2[rs], NL2 + ro, 512, &S.rfull[rs]);
                bulk_load(S.dd[rs], Drow + ro, 512, &S.rfull[rs]);
            }
        }
    } else if (warp == 1) {
        if (nw > 0) {
            const bool leader = elect_one();
            const uint32_t idT = idesc_bf16(128, 128, false, false);   // S^T, dP^T: both K-major
            const uint32_t idMN = idesc_bf16(128, 128, false, true);   // dV, dK: B MN-major
            const uint64_t kd = sw128_desc(smem_u32(S.k), 16, 1024);
            const uint64_t vd = sw128_desc(smem_u32(S.v), 16, 1024);
            // stage 0 of Q and dO as K-major (B of S^T, dP^T) and MN-major (B of dK, dV)
            const uint64_t qk0 = sw128_desc(smem_u32(S.q[0]), 16, 1024);
            const uint64_t ok0 = sw128_desc(smem_u32(S.dout[0]), 16, 1024);
            const uint64_t qm0 = sw128_desc(smem_u32(S.q[0]), kTile / 2, 1024);
            const uint64_t om0 = sw128_desc(smem_u32(S.dout[0]), kTile / 2, 1024);
            // S^T(n) = K Q(n)^T and dP^T(n) = V dO(n)^T
            auto issue_st = [&](int n) -> bool {
                const int qs = n % kDkvQStages;
                if (!warp_wait(&S.qfull[qs], (n / kDkvQStages) & 1, abort, status)) return false;
                tc_fence_after();
                const uint64_t bd = desc_add(qk0, qs * kTile);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTile / 2) + (kk & 3) * 32;
                    if (leader) mma_ss(tmem + cST, desc_add(kd, off), desc_add(bd, off), idT, kk > 0);
                }
                if (leader) mma_commit(&S.st_full);
                return true;
            };
            auto issue_dp = [&](int n) -> bool {
                const int os = n % kDkvOStages;
                if (!warp_wait(&S.ofull[os], (n / kDkvOStages) & 1, abort, status)) return false;
                tc_fence_after();
                const uint64_t bd = desc_add(ok0, os * kTile);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTile / 2) + (kk & 3) * 32;
                    if (leader) mma_ss(tmem + cDP, desc_add(vd, off), desc_add(bd, off), idT, kk > 0);
                }
                if (leader) mma_commit(&S.dp_full);
                return true;
            };
            bool ok = warp_wait(&S.kv_full, 0, abort, status) && issue_st(0) && issue_dp(0);
            for (int n = 0; ok && n < nw; ++n) {
                const uint64_t qm = desc_add(qm0, (n % kDkvQStages) * kTile);
                const uint64_t om = desc_add(om0, (n % kDkvOStages) * kTile);
                const uint32_t acc = n > 0 ? 1u : 0u;
                // dV(n) in two halves, each issued once the elementwise warps stored the
                // first (k-steps 0, 2, 4, 6) or second 16 rows of every 32-row part
                bool okh = true;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (!warp_wait(&S.p_ready[h], n & 1, abort, status)) {
                        okh = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = h; kk < 8; kk += 2)
                        if (leader)
                            mma_ts(tmem + cDV, tmem + cST + part_col(kk), desc_add(om, kk * 2048), idMN,
                                   kk > 0 ? 1u : acc);
                }
                if (!okh) break;
                if (leader) mma_commit(&S.oempty[n % kDkvOStages]);
                const bool more = n + 1 < nw;
                if (more && !issue_st(n + 1)) break;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (!warp_wait(&S.ds_ready[h], n & 1, abort, status)) {
                        okh = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = h; kk < 8; kk += 2)
                        if (leader)
                            mma_ts(tmem + cDK, tmem + cDP + part_col(kk), desc_add(qm, kk * 2048), idMN,
                                   kk > 0 ? 1u : acc);
                }
                if (!okh) break;
                if (leader) mma_commit(&S.qempty[n % kDkvQStages]);
                if (more && !issue_dp(n + 1)) break;
            }
            if (leader) mma_commit(&S.acc_done);
            if (leader) mma_commit(&S.fin);
            wait_done(&S.fin, 0);
        }
    } else {
        // thread = key row c (TMEM lane); part p takes query rows 32p..32p+31 of each item
        const int quad = warp & 3, part = (warp - 2) >> 2;
        const int c = quad * 32 + lane;
        const int j = k0 + c;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t colS = cST + part * 32, colP = cDP + part * 32;
        const int32_t kap = j < N ? m.kappa[(int64_t)b * N + j] : 0;
        bool ok = true;
        for (int n = 0; n < nw; ++n) {
            const int s = n % kDkvRowStages;
            const uint32_t ph = n & 1;
            if (!warp_wait(&S.rfull[s], (n / kDkvRowStages) & 1, abort, status)) {
                ok = false;
                break;
            }
            const int q0 = S.q0[s] + 32 * part;  // this part's first row
            // visible query rows of this key among the part's 32: [rlo, rhi) (j <= t < kappa_j)
            int rlo = 0, rhi = 32;
            if (!S.full_tile[s]) {
                if (j >= N) {
                    rlo = rhi = 0;
                } else {
                    const int64_t lo = (int64_t)j - q0, hi = (int64_t)(kap < N ? kap : N) - q0;
                    rlo = (int)(lo < 0 ? 0 : (lo > 32 ? 32 : lo));
                    rhi = (int)(hi < 0 ? 0 : (hi > 32 ? 32 : hi));
                }
            }
            if (!warp_wait(&S.st_full, ph, abort, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // P^T = 2^(S^T c - LSE_t log2 e), kept in fp32 for dS^T and stored as
            // bf16 pairs (the A operand of dV)
            float pf[32];
            {
                uint32_t r0[32];
                tmem_ld32(tmem + lane_off + colS, r0);
                tmem_ld_wait();
                const float4 *l2v = reinterpret_cast<const float4 *>(S.nl2[s] + 32 * part);
                const bool masked = __any_sync(0xffffffffu, rlo > 0 || rhi < 32);
                // in two halves of 16 rows, each handed to the MMA warp as soon as stored
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int i = 4 * h; i < 4 * h + 4; ++i) {
                        const float4 lv = l2v[i];
                        // a quarter of the exponentials on the FMA pipe, the rest on the SFU
                        float x0, x1, x2, x3;
                        fma2v(__uint_as_float(r0[4 * i]), __uint_as_float(r0[4 * i + 1]), scale_log2, lv.x,
                              lv.y, x0, x1);
                        fma2v(__uint_as_float(r0[4 * i + 2]), __uint_as_float(r0[4 * i + 3]), scale_log2, lv.z,
                              lv.w, x2, x3);
                        if (i & 1) {
                            exp2_fma_x2(x0, x1, pf[4 * i], pf[4 * i + 1]);
                        } else {
                            pf[4 * i] = ex2(x0);
                            pf[4 * i + 1] = ex2(x1);
                        }
                        pf[4 * i + 2] = ex2(x2);
                        pf[4 * i + 3] = ex2(x3);
                    }
                    if (masked) {
#pragma unroll
                        for (int rr = 16 * h; rr < 16 * h + 16; ++rr)
                            pf[rr] = (rr >= rlo && rr < rhi) ? pf[rr] : 0.f;
                    }
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(pf[16 * h + 2 * i], pf[16 * h + 2 * i + 1]);
                    tmem_st8(tmem + lane_off + colS + 8 * h, pk);
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(&S.p_ready[h]);
                }
            }
            if (!warp_wait(&S.dp_full, ph, abort, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // dS^T = P^T (dP^T - D_t), in the same two halves
            {
                uint32_t r0[32];
                tmem_ld32(tmem + lane_off + colP, r0);
                tmem_ld_wait();
                const float4 *ddv = reinterpret_cast<const float4 *>(S.dd[s] + 32 * part);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t dk2[8];
#pragma unroll
                    for (int i = 4 * h; i < 4 * h + 4; ++i) {
                        const float4 dv4 = ddv[i];
                        float d0, d1, d2, d3;
                        f2_split(f2_mul(f2_make(pf[4 * i], pf[4 * i + 1]),
                                        f2_sub(f2_make(__uint_as_float(r0[4 * i]), __uint_as_float(r0[4 * i + 1])),
                                               f2_make(dv4.x, dv4.y))), d0, d1);
                        f2_split(f2_mul(f2_make(pf[4 * i + 2], pf[4 * i + 3]),
                                        f2_sub(f2_make(__uint_as_float(r0[4 * i + 2]), __uint_as_float(r0[4 * i + 3])),
                                               f2_make(dv4.z, dv4.w))), d2, d3);
                        dk2[2 * (i - 4 * h)] = pack_bf16(d0, d1);
                        dk2[2 * (i - 4 * h) + 1] = pack_bf16(d2, d3);
                    }
                    tmem_st8(tmem + lane_off + colP + 8 * h, dk2);
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(&S.ds_ready[h]);
                }
            }
            mbar_arrive(&S.rempty[s]);  // done with this item's row data
        }
        // each part writes 32 of the 128 dimensions of dV and dK
        const uint32_t col0 = part * 32;
        if (ok && nw > 0 && warp_wait(&S.acc_done, 0, abort, status)) {
            tc_fence_after();
            const int64_t ro = (((int64_t)b * N + j) * Hkv + kvh) * 128 + col0;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                uint32_t r0[32];
                const float f = which ? scale : 1.f;
                tmem_ld32(tmem + lane_off + (which ? cDK : cDV) + col0, r0);
                tmem_ld_wait();
                if (j < N) store_row32((which ? dk : dv) + ro, r0, f);
            }
        } else if (nw == 0 && j < N) {
            // a key no query sees (cannot happen for a valid mask: the diagonal is visible)
            const int64_t ro = (((int64_t)b * N + j) * Hkv + kvh) * 128 + col0;
            for (int i = 0; i < 32; i += 8) {
                *reinterpret_cast<uint4 *>(dk + ro + i) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(dv + ro + i) = make_uint4(0, 0, 0, 0);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------- dQ
//
// TMEM: S [0,128), dP [128,256), dQ accumulator [256,384), and the CTA's Q
// [384,448) and dO [448,512) as bf16 pairs: S = Q K^T and dP = dO V^T take
// their A operand from TMEM, so each product reads only K or V from shared
// memory (160 KB of shared-memory reads and fills per item instead of 224 KB,
// below the 1536 cycles of tensor work). Sixteen elementwise warps (four per
// TMEM lane quarter, so that each scheduler has four to hide the TMEM and
// exponential latencies) split an item's 128 keys in four parts of 32 (thread =
// query row); each writes its dS as bf16 pairs into the first 16 of its own 32
// columns of dP, the A operand of dQ += dS K. Per item the tensor core runs, in issue order, dP(n),
// [S(n) read] S(n+1), [dS(n) written] dQ(n), then dP(n+1): each product that
// overwrites a TMEM region comes after the one that reads it.
//
// K is needed from S_n until dQ_n, V only for dP_n. K has three stages (the
// load of K_{n+2} goes out when dQ_{n-1} completes, 2048 cycles of tensor work
// before S_{n+2}), V two (V_{n+2} when dP_n completes, five products ahead).
constexpr int kDqKStages = 3;
constexpr int kDqVStages = 2;

struct DqSmem {
    uint8_t k[kDqKStages][kTile];
    uint8_t v[kDqVStages][kTile];
    uint32_t bits[kDqKStages][128 * 4];  // mask rows of the key tile in each K stage (partial tiles)
    int32_t pid[kDqKStages];             // its partial index (-1: full)
    uint64_t kfull[kDqKStages], kempty[kDqKStages], vfull[kDqVStages], vempty[kDqVStages], qo_ready,
        s_full, dp_full, s_free, ds_ready, acc_done, fin;
    uint32_t tmem_base;
    int abort;
};

__global__ void __launch_bounds__(kBwdThreads, 1)
    k_attn_dq_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ dO,
                 kvs_tile_mask m, int32_t Hq, int32_t Hkv, float scale, float scale_log2,
                 const float *__restrict__ Drow, const float *__restrict__ NL2,
                 __nv_bfloat16 *__restrict__ dq, int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    DqSmem &S = *reinterpret_cast<DqSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = m.B, N = m.N, T = m.T, G = Hq / Hkv, Tpad = T * 128;
    const int64_t idx = blockIdx.x;
    const int qi = T - 1 - (int)(idx / ((int64_t)B * Hq));
    const int rem = (int)(idx % ((int64_t)B * Hq));
    const int hq = rem % Hq, b = rem / Hq, kvh = hq / G;
    const int q0 = qi * 128;
    const int32_t e0 = m.row_ptr[b * T + qi], nt = m.row_ptr[b * T + qi + 1] - e0;
    if (grid_timed_out(status)) return;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDqKStages; ++i) {
            mbar_init(&S.kfull[i], 1);
            mbar_init(&S.kempty[i], 1);
        }
        for (int i = 0; i < kDqVStages; ++i) {
            mbar_init(&S.vfull[i], 1);
            mbar_init(&S.vempty[i], 1);
        }
        mbar_init(&S.qo_ready, kBwdEwThreads);
        mbar_init(&S.s_full, 1);
        mbar_init(&S.dp_full, 1);
        mbar_init(&S.s_free, kBwdEwThreads);
        mbar_init(&S.ds_ready, kBwdEwThreads);
        mbar_init(&S.acc_done, 1);
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
    constexpr uint32_t cS = 0, cDP = 128, cDQ = 256, cQ = 384, cO = 448;

    if (warp == 0) {
        if (lane == 0 && nt > 0) {
            for (int n = 0; n < nt; ++n) {
                const int ks = n % kDqKStages;
                const int k0 = m.row_col[e0 + n] * 128;
                if (n >= kDqKStages &&
                    !mbar_wait(&S.kempty[ks], ((n / kDqKStages) - 1) & 1, abort, status))
                    break;
                const int32_t pid = m.row_pidx[e0 + n];
                S.pid[ks] = pid;
                mbar_expect_tx(&S.kfull[ks], kTile + (pid >= 0 ? 2048u : 0u));
                tma_load_4d(S.k[ks], &tmK, &S.kfull[ks], 0, kvh, k0, b);
                tma_load_4d(S.k[ks] + kTile / 2, &tmK, &S.kfull[ks], 64, kvh, k0, b);
                if (pid >= 0) bulk_load(S.bits[ks], m.bits + (int64_t)pid * 512, 2048, &S.kfull[ks]);
                const int vs = n % kDqVStages;
                if (n >= kDqVStages &&
                    !mbar_wait(&S.vempty[vs], ((n / kDqVStages) - 1) & 1, abort, status))
                    break;
                mbar_expect_tx(&S.vfull[vs], kTile);
                tma_load_4d(S.v[vs], &tmV, &S.vfull[vs], 0, kvh, k0, b);
                tma_load_4d(S.v[vs] + kTile / 2, &tmV, &S.vfull[vs], 64, kvh, k0, b);
            }
        }
    } else if (warp == 1) {
        if (nt > 0) {
            const bool leader = elect_one();
            const uint32_t idKM = idesc_bf16(128, 128, false, false);
            const uint32_t idMN = idesc_bf16(128, 128, false, true);
            const uint64_t kd0 = sw128_desc(smem_u32(S.k[0]), 16, 1024);         // + stage * kTile
            const uint64_t km0 = sw128_desc(smem_u32(S.k[0]), kTile / 2, 1024);  // MN-major view
            const uint64_t vd0 = sw128_desc(smem_u32(S.v[0]), 16, 1024);         // + stage * kTile
            // S(n) = Q K(n)^T, A = Q from TMEM (d in bf16 pairs: K step kk at column 8 kk)
            auto issue_s = [&](int n) -> bool {
                const int ks = n % kDqKStages;
                if (!warp_wait(&S.kfull[ks], (n / kDqKStages) & 1, abort, status)) return false;
                tc_fence_after();
                const uint64_t kd = desc_add(kd0, ks * kTile);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTile / 2) + (kk & 3) * 32;
                    if (leader) mma_ts(tmem + cS, tmem + cQ + 8 * kk, desc_add(kd, off), idKM, kk > 0);
                }
                if (leader) mma_commit(&S.s_full);
                return true;
            };
            // dP(n) = dO V(n)^T, A = dO from TMEM
            auto issue_dp = [&](int n) -> bool {
                const int vs = n % kDqVStages;
                if (!warp_wait(&S.vfull[vs], (n / kDqVStages) & 1, abort, status)) return false;
                tc_fence_after();
                const uint64_t vd = desc_add(vd0, vs * kTile);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * (kTile / 2) + (kk & 3) * 32;
                    if (leader) mma_ts(tmem + cDP, tmem + cO + 8 * kk, desc_add(vd, off), idKM, kk > 0);
                }
                if (leader) mma_commit(&S.dp_full);
                if (leader) mma_commit(&S.vempty[vs]);
                return true;
            };
            bool ok = warp_wait(&S.qo_ready, 0, abort, status);
            if (ok) {
                tc_fence_after();
                ok = issue_s(0) && issue_dp(0);
            }
            for (int n = 0; ok && n < nt; ++n) {
                const bool more = n + 1 < nt;
                // S(n+1) overwrites S(n) once the elementwise warps have read it
                if (more) {
                    if (!warp_wait(&S.s_free, n & 1, abort, status)) break;
                    if (!issue_s(n + 1)) break;
                }
                // dQ(n) += dS(n) K(n), dS in the dP columns
                if (!warp_wait(&S.ds_ready, n & 1, abort, status)) break;
                tc_fence_after();
                const uint64_t km = desc_add(km0, (n % kDqKStages) * kTile);
                const uint32_t acc = n > 0 ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    if (leader)
                        mma_ts(tmem + cDQ, tmem + cDP + part_col(kk), desc_add(km, kk * 2048), idMN,
                               kk > 0 ? 1u : acc);
                if (leader) mma_commit(&S.kempty[n % kDqKStages]);
                // dP(n+1) overwrites dS(n) after dQ(n) has read it (in issue order)
                if (more && !issue_dp(n + 1)) break;
            }
            if (leader) mma_commit(&S.acc_done);
            if (leader) mma_commit(&S.fin);
            wait_done(&S.fin, 0);
        }
    } else {
        // thread = query row (TMEM lane); part = which 32 key columns (and which 32
        // dimensions of Q, dO and dQ) it handles
        const int quad = warp & 3, part = (warp - 2) >> 2;
        const int row = quad * 32 + lane;
        const int t = q0 + row;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t col0 = part * 32;
        const int64_t ro = ((int64_t)b * Hq + hq) * Tpad + t;
        const float nl2 = NL2[ro], dd = Drow[ro];
        const uint64_t dd2 = f2_make(dd, dd);
        bool ok = true;
        if (nt > 0) {
            // this row's part of Q and of dO into TMEM as bf16 pairs (the A operands);
            // rows past N are zero
            uint32_t r[16];
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const __nv_bfloat16 *src = (w ? dO : q) + (((int64_t)b * N + t) * Hq + hq) * 128 + col0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 u = t < N ? *reinterpret_cast<const uint4 *>(src + 8 * i) : make_uint4(0, 0, 0, 0);
                    r[4 * i] = u.x;
                    r[4 * i + 1] = u.y;
                    r[4 * i + 2] = u.z;
                    r[4 * i + 3] = u.w;
                }
                tmem_st16(tmem + lane_off + (w ? cO : cQ) + part * 16, r);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&S.qo_ready);
        }
        for (int n = 0; n < nt; ++n) {
            // the K stage carries the tile's mask rows; it is refilled only after
            // dQ_n, i.e. after this item's dS
            const int ks = n % kDqKStages;
            if (!warp_wait(&S.kfull[ks], (n / kDqKStages) & 1, abort, status)) {
                ok = false;
                break;
            }
            const bool partial = S.pid[ks] >= 0;  // same for the whole CTA
            const uint32_t bits = partial ? S.bits[ks][row * 4 + part] : ~0u;
            if (!warp_wait(&S.s_full, n & 1, abort, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // P = 2^(S c - LSE log2 e) for this thread's 32 key columns, kept in fp32;
            // dS = P (dP - D) then rounds to bf16 for the dQ MMA
            float pf[32];
            {
                uint32_t r0[32];
                tmem_ld32(tmem + lane_off + cS + col0, r0);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&S.s_free);
#pragma unroll
                for (int jj = 0; jj < 32; jj += 4) {
                    // a quarter of the exponentials on the FMA pipe, the rest on the SFU
                    float x0, x1, x2, x3;
                    fma2(__uint_as_float(r0[jj]), __uint_as_float(r0[jj + 1]), scale_log2, nl2, x0, x1);
                    fma2(__uint_as_float(r0[jj + 2]), __uint_as_float(r0[jj + 3]), scale_log2, nl2, x2, x3);
                    if ((jj >> 2) & 1) {
                        exp2_fma_x2(x0, x1, pf[jj], pf[jj + 1]);
                    } else {
                        pf[jj] = ex2(x0);
                        pf[jj + 1] = ex2(x1);
                    }
                    pf[jj + 2] = ex2(x2);
                    pf[jj + 3] = ex2(x3);
                }
                if (partial) {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) pf[jj] = ((bits >> jj) & 1u) ? pf[jj] : 0.f;
                }
            }
            if (!warp_wait(&S.dp_full, n & 1, abort, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                uint32_t r0[32], pk[16];
                tmem_ld32(tmem + lane_off + cDP + col0, r0);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < 32; jj += 2) {
                    float d0, d1;
                    f2_split(f2_mul(f2_make(pf[jj], pf[jj + 1]),
                                    f2_sub(f2_make(__uint_as_float(r0[jj]), __uint_as_float(r0[jj + 1])), dd2)),
                             d0, d1);
                    pk[jj >> 1] = pack_bf16(d0, d1);
                }
                // keys col0..col0+31 as bf16 pairs in the first 16 columns of this part
                tmem_st16(tmem + lane_off + cDP + col0, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&S.ds_ready);
        }
        if (ok && nt > 0 && warp_wait(&S.acc_done, 0, abort, status)) {
            tc_fence_after();
            uint32_t r0[32];
            tmem_ld32(tmem + lane_off + cDQ + col0, r0);
            tmem_ld_wait();
            if (t < N) store_row32(dq + (((int64_t)b * N + t) * Hq + hq) * 128 + col0, r0, scale);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t bwd_tc_ws_bytes(int32_t B, int32_t N, int32_t Hq) {
    const int64_t Tpad = (int64_t)((N + 127) / 128) * 128;
    return 2 * (size_t)B * Hq * Tpad * sizeof(float);
}

cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const void *o,
                          const void *o_lo, const void *dO, const float *lse, const kvs_tile_mask &m, int32_t Hq,
                          int32_t Hkv, float scale, void *dq, void *dk, void *dv, void *ws,
                          int32_t stages, int32_t *status, cudaStream_t s, bool *map_ok) {
    CUtensorMap tq, tk, tv, to;
    *map_ok = make_tmap_bnhd(&tq, q, m.B, m.N, Hq, 128) && make_tmap_bnhd(&tk, k, m.B, m.N, Hkv, 128) &&
              make_tmap_bnhd(&tv, v, m.B, m.N, Hkv, 128) && make_tmap_bnhd(&to, dO, m.B, m.N, Hq, 128);
    if (!*map_ok) return cudaSuccess;
    const int32_t Tpad = m.T * 128;
    float *Drow = (float *)ws;
    float *NL2 = Drow + (size_t)m.B * Hq * Tpad;
    const int64_t rows = (int64_t)m.B * Hq * Tpad;
    if (stages & KVS_BWD_PREP)
        k_bwd_prep<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
            (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)o_lo, (const __nv_bfloat16 *)dO, lse,
            m.B, m.N, Hq, Tpad, Drow, NL2);
    const float sl2 = scale * 1.4426950408889634f;
    cudaError_t e = cudaSuccess;
    if (stages & KVS_BWD_DKDV) {
        const size_t smem = sizeof(DkvSmem);
        e = cudaFuncSetAttribute(k_attn_dkdv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        k_attn_dkdv_tc<<<(unsigned)((int64_t)m.B * Hkv * m.T), kBwdThreads, smem, s>>>(
            tq, tk, tv, to, m, Hq, Hkv, scale, sl2, Drow, NL2, (__nv_bfloat16 *)dk,
            (__nv_bfloat16 *)dv, status);
    }
    if (stages & KVS_BWD_DQ) {
        const size_t smem = sizeof(DqSmem) + 1024;
        e = cudaFuncSetAttribute(k_attn_dq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        k_attn_dq_tc<<<(unsigned)((int64_t)m.B * Hq * m.T), kBwdThreads, smem, s>>>(
            tk, tv, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)dO, m, Hq, Hkv, scale, sl2, Drow,
            NL2, (__nv_bfloat16 *)dq, status);
    }
    return cudaGetLastError();
}

}  // namespace kvs
