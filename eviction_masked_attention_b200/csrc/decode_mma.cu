// bf16 split-K paged decode: cp.async staging of the live K/V rows into shared
// memory, warp-level tensor-core MMAs for the small per-token products.
//
// "KV-streams: speeding up agentic RL by operating on the KV cache directly":
// generation continues from the entries that survived compaction; the cache
// is paged (16-token or 1-token blocks) and read through a block table without
// holes.
//
// The CTAs share the step's live entries equally (decode_sched.cuh): a CTA
// streams one or more pieces, each a contiguous range of live entries of one
// (sequence, kv head) unit, for all G query heads that share the kv head, so
// every K/V byte is read from HBM once. For a piece, each of the 4 warps takes
// 16-entry chunks w, w+4, ... and keeps a 2-stage ring of them in flight: its lanes copy the
// 256-byte key and value rows (found through the block table slice held in
// shared memory; a 16-token block is 16 consecutive rows, with 1-token blocks
// every row comes from its own slot) in 16-byte cp.async pieces into rows of
// 272 bytes, so ldmatrix reads are free of bank conflicts. Per chunk it computes
//   S (G x 16) = Q K^T     mma.m16n8k16, Q in registers (G <= 8; rows >= G zero)
//   online softmax in base 2 on the accumulator fragments
//   O (G x 128) += P V     P re-used from the S fragments as the A operand
// Per-warp states merge in shared memory; a piece that is a whole unit writes
// the output, any other writes its partial (max, sum, unnormalised output) and
// the merge kernel folds the partials of a unit.
#include <algorithm>

#include "decode_sched.cuh"

namespace kvs {

constexpr int kDmWarps = 4;      // each warp streams and computes its own chunks
constexpr int kDmStages = 2;     // ring depth per warp (2: three CTAs fit on an SM)
constexpr int kDmRow = 272;      // staged row stride in bytes (256 + 16)
constexpr int kDmChunk = 16;     // entries per stage
constexpr int kDmThreads = 32 * kDmWarps;
constexpr int kDmMaxTps = kDecMaxChunksPerCta * kDecChunk;  // entries of one piece (at most)
static_assert(kDmThreads == kDecThreads && kDmChunk == kDecChunk, "decode work split");

struct DmSmem {
    uint8_t k[kDmWarps][kDmStages][kDmChunk * kDmRow];
    uint8_t v[kDmWarps][kDmStages][kDmChunk * kDmRow];
    float m[kDmWarps][16], l[kDmWarps][16];
    int32_t blk[kDmMaxTps + 16];  // this piece's slice of the block table
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D = A (16x16 bf16, row) * B (16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// K/V rows are read once per call: they enter L2 as the first lines to evict, so the
// stream does not push out what the kernels before the decode left there (a step's
// last kernels leave L2 full of lines still to be written back)
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// BS is the block size when it is one the workloads use (16: a chunk is one whole
// block; 1: one block per entry), 0 for any other; it only shortens the address
// arithmetic of the copies.
template <int G, int BS>
__global__ void __launch_bounds__(kDmThreads, 3)
    k_decode_mma(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kc,
                 const __nv_bfloat16 *__restrict__ vc, const int32_t *__restrict__ block_table,
                 const int32_t *__restrict__ num_tokens, int32_t B, int32_t Hq, int32_t Hkv,
                 int32_t bs, int32_t max_blocks, int32_t pool_blocks, float scale_log2,
                 int64_t n_cta, int64_t *pre_ws, float *partials, __nv_bfloat16 *__restrict__ o,
                 int32_t *status) {
    static_assert(G >= 1 && G <= 8, "query heads per kv head (rows 8..15 of the MMA are padding)");
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    DmSmem &S = *reinterpret_cast<DmSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                           ~uintptr_t(127));
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // max_blocks * bs fits in int32 (checked by the host); counts outside
    // [0, max_blocks * bs] are reported (by CTA 0) and clamped
    const int32_t cap = max_blocks * bs;
    const DecodeRange rg = dec_locate(num_tokens, B, Hkv, cap, n_cta, pre_ws, status);
    if (rg.x0 >= rg.x1) return;
    const int64_t blk_stride = (int64_t)Hkv * bs * D;
    const int piece = lane & 15, par = lane >> 4;
    const uint64_t pol = l2_evict_first();
    const int g = lane >> 2, t4 = lane & 3;
    // chunks of one sub-piece: its ids (at most (chunks * 16 - 1) / bs + 2 of them)
    // must fit the kDmMaxTps + 16 staged slots
    const int32_t sub_chunks = bs >= kDmChunk ? kDmMaxTps : kDecMaxChunksPerCta * max(1, bs);

    int32_t b = rg.b0;
    int32_t pre = rg.pre_b0;
    int32_t ntok = dec_ntok(num_tokens, b, cap);
    int32_t nch = dec_nch(ntok);
    int32_t kvh = (rg.x0 - Hkv * pre) / nch;
    for (;;) {
        // this piece: unit (b, kvh), chunks [ps, pe) of the unit's [cs, ce)
        const int32_t cs = Hkv * pre + kvh * nch, ce = cs + nch;
        const int32_t ps = max(rg.x0, cs), pe = min(rg.x1, ce);
        const bool whole = ps == cs && pe == ce;
        const int32_t *bt = block_table + (int64_t)b * max_blocks;
        const int64_t head_off = (int64_t)kvh * bs * D;

        // Q as the A operand: rows = query heads (rows >= G are zero), 16 dims per k-step
        uint32_t qa[8][4];
        const __nv_bfloat16 *qb = q + ((int64_t)b * Hq + (int64_t)kvh * G) * D;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c0 = 16 * kk + 2 * t4;
            qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t *>(qb + g * D + c0) : 0u;
            qa[kk][1] = g + 8 < G ? *reinterpret_cast<const uint32_t *>(qb + (g + 8) * D + c0) : 0u;
            qa[kk][2] = g < G ? *reinterpret_cast<const uint32_t *>(qb + g * D + c0 + 8) : 0u;
            qa[kk][3] = g + 8 < G ? *reinterpret_cast<const uint32_t *>(qb + (g + 8) * D + c0 + 8) : 0u;
        }
        float acc[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        float mrow = -INFINITY, lrow = 0.f;  // row g (head g); rows g+8 are padding

        // sub-pieces whose table slice fits the kDmMaxTps + 16 ids staged in shared
        // memory (72 chunks of 1-token blocks, 1152 of 16-token blocks); the softmax
        // state carries over from one to the next
        for (int32_t sp = ps; sp < pe; sp += sub_chunks) {
            const int32_t spe = min(pe, sp + sub_chunks);
            const int32_t t_begin = (sp - cs) * kDecChunk;
            const int32_t t_end = min(ntok, (spe - cs) * kDecChunk);
            const int nchunks = (t_end - t_begin + kDmChunk - 1) / kDmChunk;
            // the block ids this sub-piece needs (entries t_begin..t_end-1); an id
            // outside the pool is reported and kept as -1: its entries are never
            // copied and count as masked (score -inf, value row zero)
            const int32_t blk0 = t_begin / bs;
            const int32_t nblk = (t_end - 1) / bs - blk0 + 1;
            __syncthreads();  // the previous sub-piece is done with the slice and the rings
            for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
                int32_t id = bt[blk0 + i];
                if (id < 0 || id >= pool_blocks) {
                    set_status(status, KVS_ERR_INVALID_ARG);
                    id = -1;
                }
                S.blk[i] = id;
            }
            __syncthreads();

            // this warp's chunks are w, w + kDmWarps, ...; each lane copies 16-byte piece
            // (lane & 15) of entries (lane >> 4) + 2j, j = 0..7, for both K and V
            auto issue = [&](int i) {
                const int c = w + i * kDmWarps;
                if (c < nchunks) {
                    const int s = i % kDmStages;
                    const int32_t t0 = t_begin + c * kDmChunk;
                    const int nv = min(kDmChunk, t_end - t0);
                    const uint32_t kd = smem_u32(S.k[w][s]) + piece * 16, vd = smem_u32(S.v[w][s]) + piece * 16;
                    if constexpr (BS == kDmChunk) {
                        // sub-pieces start at multiples of 16 entries, so a chunk is exactly one block
                        const int32_t id = S.blk[t0 / kDmChunk - blk0];
                        const int64_t base = (int64_t)id * blk_stride + head_off + piece * 8;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int e = par + 2 * j;
                            if (e < nv && id >= 0) {
                                cp_async16(kd + e * kDmRow, kc + base + e * D, pol);
                                cp_async16(vd + e * kDmRow, vc + base + e * D, pol);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int e = par + 2 * j;
                            if (e < nv) {
                                const int32_t t = t0 + e;
                                const int32_t id = BS == 1 ? S.blk[t - blk0] : S.blk[t / bs - blk0];
                                const int64_t off = BS == 1 ? (int64_t)id * blk_stride + head_off + piece * 8
                                                            : (int64_t)id * blk_stride + head_off +
                                                                  (int64_t)(t % bs) * D + piece * 8;
                                if (id >= 0) {
                                    cp_async16(kd + e * kDmRow, kc + off, pol);
                                    cp_async16(vd + e * kDmRow, vc + off, pol);
                                }
                            }
                        }
                    }
                }
                cp_async_commit();  // one group per step, empty past the end
            };
#pragma unroll
            for (int i = 0; i < kDmStages - 1; ++i) issue(i);

            for (int i = 0, c = w; c < nchunks; ++i, c += kDmWarps) {
                issue(i + kDmStages - 1);
                cp_async_wait<kDmStages - 1>();  // this lane's copies of chunk i are done
                __syncwarp();                    // ... and those of the other lanes
                const int s = i % kDmStages;
                const int32_t t0 = t_begin + c * kDmChunk;
                const int nv = min(kDmChunk, t_end - t0);
                const uint32_t ks = smem_u32(S.k[w][s]), vs = smem_u32(S.v[w][s]);
                // this lane's entries 2 t4, 2 t4 + 1, 8 + 2 t4, 9 + 2 t4: inside the piece
                // and with a block id in the pool (the others were not copied)
                auto entry_ok = [&](int e) -> bool {
                    if (e >= nv) return false;
                    const int32_t t = t0 + e;
                    const int32_t id = BS == kDmChunk ? S.blk[t0 / kDmChunk - blk0]
                                                      : (BS == 1 ? S.blk[t - blk0] : S.blk[t / bs - blk0]);
                    return id >= 0;
                };
                const bool ok0 = entry_ok(2 * t4), ok1 = entry_ok(2 * t4 + 1), ok2 = entry_ok(8 + 2 * t4),
                           ok3 = entry_ok(9 + 2 * t4);
                const bool chunk_ok = __all_sync(0xffffffffu, ok0 && ok1 && ok2 && ok3);
                const bool okv[4] = {ok0, ok1, ok2, ok3};
                // S = Q K^T for entries 0..7 (j = 0) and 8..15 (j = 1)
                float sc[2][4];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
                    for (int kk = 0; kk < 8; kk += 2) {
                        uint32_t b0, b1, b2, b3;
                        const uint32_t addr = ks + (8 * j + (lane & 7)) * kDmRow + kk * 32 + (lane >> 3) * 16;
                        ldsm_x4(addr, b0, b1, b2, b3);
                        mma16816(sc[j], qa[kk], b0, b1);
                        mma16816(sc[j], qa[kk + 1], b2, b3);
                    }
                }
                // online softmax on row g: entries 8j + 2 t4 + {0, 1}
                float x[4];
                float cm = -INFINITY;
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        x[2 * j + u] = okv[2 * j + u] ? sc[j][u] * scale_log2 : -INFINITY;
                        cm = fmaxf(cm, x[2 * j + u]);
                    }
                cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
                cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
                const float mn = fmaxf(mrow, cm);
                const float mref = mn == -INFINITY ? 0.f : mn;
                const float alpha = ex2(mrow - mref);
                float p[4], psum = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    p[u] = ex2(x[u] - mref);
                    psum += p[u];
                }
                psum += __shfl_xor_sync(0xffffffffu, psum, 1);
                psum += __shfl_xor_sync(0xffffffffu, psum, 2);
                lrow = lrow * alpha + psum;
                mrow = mn;
                // P as the A operand (rows g, entries 2 t4 (+8)); padding rows stay zero
                const uint32_t pa[4] = {pack_bf16(p[0], p[1]), 0u, pack_bf16(p[2], p[3]), 0u};
                // value rows of entries that were not copied this time (past the piece's
                // end, or with an id outside the pool) hold stale data: zero them
                const bool z0 = !ok0, z1 = !ok1, z2 = !ok2, z3 = !ok3;
#pragma unroll
                for (int dt = 0; dt < 16; dt += 2) {
                    uint32_t b0, b1, b2, b3;
                    const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
                    const uint32_t addr = vs + row * kDmRow + (dt + (lane >> 4)) * 16;
                    ldsm_x4_t(addr, b0, b1, b2, b3);
                    if (!chunk_ok) {
                        b0 = (z0 ? b0 & 0xFFFF0000u : b0);
                        b0 = (z1 ? b0 & 0x0000FFFFu : b0);
                        b1 = (z2 ? b1 & 0xFFFF0000u : b1);
                        b1 = (z3 ? b1 & 0x0000FFFFu : b1);
                        b2 = (z0 ? b2 & 0xFFFF0000u : b2);
                        b2 = (z1 ? b2 & 0x0000FFFFu : b2);
                        b3 = (z2 ? b3 & 0xFFFF0000u : b3);
                        b3 = (z3 ? b3 & 0x0000FFFFu : b3);
                    }
                    acc[dt][0] *= alpha;
                    acc[dt][1] *= alpha;
                    acc[dt + 1][0] *= alpha;
                    acc[dt + 1][1] *= alpha;
                    mma16816(acc[dt], pa, b0, b1);
                    mma16816(acc[dt + 1], pa, b2, b3);
                }
                __syncwarp();  // stage s is refilled by the next iteration's issue
            }
            cp_async_wait<0>();
        }
        if (t4 == 0 && g < G) {
            S.m[w][g] = mrow;
            S.l[w][g] = lrow;
        }
        // every warp is done with its ring before the value area (which reuses the
        // K rings) is written
        __syncthreads();
        float *cacc = reinterpret_cast<float *>(&S.k[0][0][0]);  // [warps][G][128]
        if (g < G) {
#pragma unroll
            for (int dt = 0; dt < 16; ++dt) {
                float *dst = cacc + ((w * G + g) * D) + 8 * dt + 2 * t4;
                dst[0] = acc[dt][0];
                dst[1] = acc[dt][1];
            }
        }
        __syncthreads();
        const int64_t u = (int64_t)b * Hkv + kvh;
        float *part = partials + (((int64_t)blockIdx.x + u) * G) * (D + 2);  // slot c + u
        for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
            const int gg = i / D, e = i % D;
            float M = -INFINITY;
#pragma unroll
            for (int ww = 0; ww < kDmWarps; ++ww) M = fmaxf(M, S.m[ww][gg]);
            const float Mr = M == -INFINITY ? 0.f : M;
            float L = 0.f, A = 0.f;
#pragma unroll
            for (int ww = 0; ww < kDmWarps; ++ww) {
                const float f = ex2(S.m[ww][gg] - Mr);
                L += S.l[ww][gg] * f;
                A += cacc[(ww * G + gg) * D + e] * f;
            }
            if (whole) {
                o[((int64_t)b * Hq + (int64_t)kvh * G + gg) * D + e] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
            } else {
                float *pp = part + (int64_t)gg * (D + 2);
                pp[e] = A;
                if (e == 0) {
                    pp[D] = M;
                    pp[D + 1] = L;
                }
            }
        }
        if (pe >= rg.x1) break;
        __syncthreads();  // the next piece refills the rings (which hold cacc) and the slice
        // next unit: the next kv head, or the next sequence with live entries
        if (++kvh == Hkv) {
            kvh = 0;
            do {
                pre += nch;
                ++b;
                ntok = dec_ntok(num_tokens, b, cap);
                nch = dec_nch(ntok);
            } while (nch == 0);
        }
    }
}

size_t decode_mma_smem() { return sizeof(DmSmem) + 128; }

template <int G, int BS>
static cudaError_t launch_g(const void *q, const void *kc, const void *vc, const int32_t *bt,
                            const int32_t *nt, int32_t B, int32_t Hq, int32_t Hkv, int32_t bs,
                            int32_t max_blocks, int32_t pool_blocks, float scale_log2, int64_t n_cta,
                            int64_t *pre_ws, float *partials, void *o, int32_t *status,
                            cudaStream_t s) {
    const size_t smem = decode_mma_smem();
    cudaError_t e =
        cudaFuncSetAttribute(k_decode_mma<G, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_decode_mma<G, BS><<<(unsigned)n_cta, kDmThreads, smem, s>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)kc, (const __nv_bfloat16 *)vc, bt, nt, B, Hq,
        Hkv, bs, max_blocks, pool_blocks, scale_log2, n_cta, pre_ws, partials, (__nv_bfloat16 *)o,
        status);
    return cudaGetLastError();
}

cudaError_t launch_decode_mma(int G, const void *q, const void *kc, const void *vc,
                              const int32_t *bt, const int32_t *nt, int32_t B, int32_t Hq,
                              int32_t Hkv, int32_t bs, int32_t max_blocks, int32_t pool_blocks,
                              float scale_log2, int64_t n_cta, int64_t *pre_ws, float *partials,
                              void *o, int32_t *status, cudaStream_t s) {
#define KVS_DM(GG, BB)                                                                    \
    return launch_g<GG, BB>(q, kc, vc, bt, nt, B, Hq, Hkv, bs, max_blocks, pool_blocks, \
                            scale_log2, n_cta, pre_ws, partials, o, status, s)
#define KVS_DM_BS(GG)              \
    if (bs == kDmChunk) KVS_DM(GG, kDmChunk); \
    if (bs == 1) KVS_DM(GG, 1);    \
    KVS_DM(GG, 0)
    switch (G) {
        case 1: KVS_DM_BS(1);
        case 2: KVS_DM_BS(2);
        case 4: KVS_DM_BS(4);
        default: KVS_DM_BS(8);
    }
#undef KVS_DM_BS
#undef KVS_DM
}

}  // namespace kvs
