// bf16 split-K paged decode: cp.async staging of the live K/V rows into shared
// memory, warp-level tensor-core MMAs for the small per-token products.
//
// "KV-streams: speeding up agentic RL by operating on the KV cache directly":
// generation continues from the entries that survived compaction; the cache
// is paged (16-token or 1-token blocks) and read through a block table without
// holes.
//
// Grid (split, kv head, sequence); one CTA streams a contiguous range of live
// entries of one kv head for all G query heads that share it, so every K/V
// byte is read from HBM once. Each of the 4 warps takes 16-entry chunks w,
// w+4, ... and keeps a 2-stage ring of them in flight: its lanes copy the
// 256-byte key and value rows (found through the block table slice held in
// shared memory; a 16-token block is 16 consecutive rows, with 1-token blocks
// every row comes from its own slot) in 16-byte cp.async pieces into rows of
// 272 bytes, so ldmatrix reads are free of bank conflicts. Per chunk it computes
//   S (G x 16) = Q K^T     mma.m16n8k16, Q in registers (G <= 8; rows >= G zero)
//   online softmax in base 2 on the accumulator fragments
//   O (G x 128) += P V     P re-used from the S fragments as the A operand
// Per-warp states merge in shared memory; with several splits each CTA writes
// its partial (max, sum, unnormalised output) and a separate combine kernel
// merges them.
#include <algorithm>

#include "common.cuh"

namespace kvs {

constexpr int kDmWarps = 4;      // each warp streams and computes its own chunks
constexpr int kDmStages = 2;     // ring depth per warp (2: three CTAs fit on an SM)
constexpr int kDmRow = 272;      // staged row stride in bytes (256 + 16)
constexpr int kDmChunk = 16;     // entries per stage
constexpr int kDmThreads = 32 * kDmWarps;
constexpr int kDmMaxTps = 1024;  // entries per split handled by one CTA (at most)

struct DmSmem {
    uint8_t k[kDmWarps][kDmStages][kDmChunk * kDmRow];
    uint8_t v[kDmWarps][kDmStages][kDmChunk * kDmRow];
    float m[kDmWarps][16], l[kDmWarps][16];
    int32_t blk[kDmMaxTps + 16];  // this split's slice of the block table
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
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
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
__global__ void __launch_bounds__(kDmThreads)
    k_decode_mma(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kc,
                 const __nv_bfloat16 *__restrict__ vc, const int32_t *__restrict__ block_table,
                 const int32_t *__restrict__ num_tokens, int32_t Hq, int32_t Hkv, int32_t bs,
                 int32_t max_blocks, float scale_log2, int32_t tps, int32_t max_splits,
                 __nv_bfloat16 *__restrict__ o, float *partials, int32_t *status) {
    static_assert(G >= 1 && G <= 8, "query heads per kv head (rows 8..15 of the MMA are padding)");
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    DmSmem &S = *reinterpret_cast<DmSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                           ~uintptr_t(127));
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t ntok = min(max(num_tokens[b], 0), max_blocks * bs);
    const int32_t nsplit = max(1, (ntok + tps - 1) / tps);
    if (split >= nsplit) return;
    const int32_t t_begin = split * tps, t_end = min(ntok, t_begin + tps);
    const int nchunks = t_end > t_begin ? (t_end - t_begin + kDmChunk - 1) / kDmChunk : 0;

    // the block ids this split needs, fetched once (entries t_begin..t_end-1)
    const int32_t *bt = block_table + (int64_t)b * max_blocks;
    const int32_t blk0 = t_begin / bs;
    const int32_t nblk = t_end > t_begin ? (t_end - 1) / bs - blk0 + 1 : 0;
    for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
        int32_t id = bt[blk0 + i];
        if (id < 0) {
            set_status(status, KVS_ERR_INVALID_ARG);
            id = 0;
        }
        S.blk[i] = id;
    }
    __syncthreads();
    const int64_t blk_stride = (int64_t)Hkv * bs * D, head_off = (int64_t)kvh * bs * D;

    // this warp's chunks are w, w + kDmWarps, ...; each lane copies 16-byte piece
    // (lane & 15) of entries (lane >> 4) + 2j, j = 0..7, for both K and V
    const int piece = lane & 15, par = lane >> 4;
    auto issue = [&](int i) {
        const int c = w + i * kDmWarps;
        if (c < nchunks) {
            const int s = i % kDmStages;
            const int32_t t0 = t_begin + c * kDmChunk;
            const int nv = min(kDmChunk, t_end - t0);
            const uint32_t kd = smem_u32(S.k[w][s]) + piece * 16, vd = smem_u32(S.v[w][s]) + piece * 16;
            if constexpr (BS == kDmChunk) {
                // splits start at multiples of 128 entries, so a chunk is exactly one block
                const int64_t base = (int64_t)S.blk[t0 / kDmChunk - blk0] * blk_stride + head_off + piece * 8;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = par + 2 * j;
                    if (e < nv) {
                        cp_async16(kd + e * kDmRow, kc + base + e * D);
                        cp_async16(vd + e * kDmRow, vc + base + e * D);
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = par + 2 * j;
                    if (e < nv) {
                        const int32_t t = t0 + e;
                        const int64_t off =
                            BS == 1 ? (int64_t)S.blk[t - blk0] * blk_stride + head_off + piece * 8
                                    : (int64_t)S.blk[t / bs - blk0] * blk_stride + head_off +
                                          (int64_t)(t % bs) * D + piece * 8;
                        cp_async16(kd + e * kDmRow, kc + off);
                        cp_async16(vd + e * kDmRow, vc + off);
                    }
                }
            }
        }
        cp_async_commit();  // one group per step, empty past the end
    };

    const int g = lane >> 2, t4 = lane & 3;
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
#pragma unroll
    for (int i = 0; i < kDmStages - 1; ++i) issue(i);

    float acc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float mrow = -INFINITY, lrow = 0.f;  // row g (head g); rows g+8 are padding
    for (int i = 0, c = w; c < nchunks; ++i, c += kDmWarps) {
        issue(i + kDmStages - 1);
        cp_async_wait<kDmStages - 1>();  // this lane's copies of chunk i are done
        __syncwarp();                    // ... and those of the other lanes
        const int s = i % kDmStages;
        const int nv = min(kDmChunk, t_end - (t_begin + c * kDmChunk));
        const uint32_t ks = smem_u32(S.k[w][s]), vs = smem_u32(S.v[w][s]);
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
                const int e = 8 * j + 2 * t4 + u;
                x[2 * j + u] = e < nv ? sc[j][u] * scale_log2 : -INFINITY;
                cm = fmaxf(cm, x[2 * j + u]);
            }
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
        const float mn = fmaxf(mrow, cm);
        const float mref = mn == -INFINITY ? 0.f : mn;
        const float alpha = ex2(mrow - mref);
        float p[4], ps = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            p[u] = ex2(x[u] - mref);
            ps += p[u];
        }
        ps += __shfl_xor_sync(0xffffffffu, ps, 1);
        ps += __shfl_xor_sync(0xffffffffu, ps, 2);
        lrow = lrow * alpha + ps;
        mrow = mn;
        // P as the A operand (rows g, entries 2 t4 (+8)); padding rows stay zero
        const uint32_t pa[4] = {pack_bf16(p[0], p[1]), 0u, pack_bf16(p[2], p[3]), 0u};
        // entries >= nv of the value rows were not copied this time: zero them
        const bool z0 = 2 * t4 >= nv, z1 = 2 * t4 + 1 >= nv, z2 = 8 + 2 * t4 >= nv,
                   z3 = 9 + 2 * t4 >= nv;
#pragma unroll
        for (int dt = 0; dt < 16; dt += 2) {
            uint32_t b0, b1, b2, b3;
            const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
            const uint32_t addr = vs + row * kDmRow + (dt + (lane >> 4)) * 16;
            ldsm_x4_t(addr, b0, b1, b2, b3);
            if (nv < kDmChunk) {
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
    const bool single = nsplit == 1;
    float *part = partials + (((int64_t)b * Hq + (int64_t)kvh * G) * max_splits) * (D + 2);
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
        if (single) {
            o[((int64_t)b * Hq + (int64_t)kvh * G + gg) * D + e] = __float2bfloat16_rn(L > 0.f ? A / L : 0.f);
        } else {
            float *pp = part + ((int64_t)gg * max_splits + split) * (D + 2);
            pp[e] = A;
            if (e == 0) {
                pp[D] = M;
                pp[D + 1] = L;
            }
        }
    }
}

size_t decode_mma_smem() { return sizeof(DmSmem) + 128; }

template <int G, int BS>
static cudaError_t launch_g(const void *q, const void *kc, const void *vc, const int32_t *bt,
                            const int32_t *nt, int32_t B, int32_t Hq, int32_t Hkv, int32_t bs,
                            int32_t max_blocks, float scale_log2, int32_t tps, int32_t max_splits,
                            void *o, float *partials, int32_t *status, cudaStream_t s) {
    const size_t smem = decode_mma_smem();
    cudaError_t e =
        cudaFuncSetAttribute(k_decode_mma<G, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(max_splits, Hkv, B);
    k_decode_mma<G, BS><<<grid, kDmThreads, smem, s>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)kc, (const __nv_bfloat16 *)vc, bt, nt, Hq,
        Hkv, bs, max_blocks, scale_log2, tps, max_splits, (__nv_bfloat16 *)o, partials, status);
    return cudaGetLastError();
}

cudaError_t launch_decode_mma(int G, const void *q, const void *kc, const void *vc,
                              const int32_t *bt, const int32_t *nt, int32_t B, int32_t Hq,
                              int32_t Hkv, int32_t bs, int32_t max_blocks, float scale_log2,
                              int32_t tps, int32_t max_splits, void *o, float *partials,
                              int32_t *status, cudaStream_t s) {
#define KVS_DM(GG, BB)                                                                               \
    return launch_g<GG, BB>(q, kc, vc, bt, nt, B, Hq, Hkv, bs, max_blocks, scale_log2, tps, max_splits, \
                            o, partials, status, s)
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
