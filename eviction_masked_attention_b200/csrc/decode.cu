// Split-K paged decode over a compacted block table.
//
// "KV-streams: speeding up agentic RL by operating on the KV cache directly":
// generation continues from the cache entries that survived compaction; the
// cache is paged (16-token blocks, or 1-token blocks) and found through a
// block table without holes, which the attention walks in order.
//
// Grid (split, kv head, sequence). A CTA streams a contiguous range of the
// sequence's live entries for one kv head and all G = Hq/Hkv query heads that
// share it (each K/V byte is read from HBM once). Each warp takes 16-entry
// chunks: lanes (2 per entry) dot 128-byte halves of the key rows with the
// queries held in shared memory, the warp runs an online softmax (base-2,
// pre-scaled logits), and lanes (16 per row, 2 rows at a time) accumulate
// 16-byte slices of the value rows. Warp states merge in shared memory; with
// several splits, each CTA writes its partial and k_decode_combine merges them.
#include <algorithm>

#include "common.cuh"

namespace kvs {

constexpr int kDecWarps = 4;

template <typename T>
struct Row16;  // unpack 16 bytes to floats
template <>
struct Row16<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ static void unpack(const uint4 &u, float (&f)[8]) {
        f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
        f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
    }
};
template <>
struct Row16<float> {
    static constexpr int E = 4;
    __device__ static void unpack(const uint4 &u, float (&f)[4]) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
};

__device__ __forceinline__ void store_out(float *o, int i, float v) { o[i] = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *o, int i, float v) {
    o[i] = __float2bfloat16_rn(v);
}

// ws: partials [B][Hq][max_splits][D + 2] fp32 (unnormalised output, max, sum)
template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32)
    k_decode(const T *__restrict__ q, const T *__restrict__ kc, const T *__restrict__ vc,
             const int32_t *__restrict__ block_table, const int32_t *__restrict__ num_tokens,
             int32_t Hq, int32_t Hkv, int32_t bs, int32_t max_blocks, float qscale, int32_t tps,
             int32_t max_splits, T *__restrict__ o, float *partials, int32_t *status) {
    using R = Row16<T>;
    constexpr int E = R::E;           // elements per 16 bytes
    static_assert(D * sizeof(T) == 256, "rows are 256 bytes");
    constexpr int HALF16 = 8;         // 16-byte pieces per half row
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t ntok = min(max(num_tokens[b], 0), max_blocks * bs);
    const int32_t nsplit = max(1, (ntok + tps - 1) / tps);
    if (split >= nsplit) return;

    __shared__ __align__(16) float s_q[G][D];
    __shared__ __align__(16) float s_p[kDecWarps][16][G];
    __shared__ float s_m[kDecWarps][G], s_l[kDecWarps][G];
    __shared__ __align__(16) float s_acc[kDecWarps][G][D];

    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, e = i % D;
        s_q[g][e] = (float)q[((int64_t)b * Hq + kvh * G + g) * D + e] * qscale;
    }
    __syncthreads();

    const int32_t t_begin = split * tps, t_end = min(ntok, t_begin + tps);
    const int32_t *bt = block_table + (int64_t)b * max_blocks;
    const int64_t head_off = (int64_t)kvh * bs * D;
    const int64_t blk_stride = (int64_t)Hkv * bs * D;

    float m[G], l[G], acc[G][E];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[g][e] = 0.f;
    }
    const int ktok = lane >> 1, khalf = lane & 1;  // key phase: entry, half row
    const int vpiece = lane & 15, vpar = lane >> 4;  // value phase: 16-B piece, entry parity

    int32_t c0 = t_begin + warp * 16;
    int32_t my_blk = -1;
    if (c0 < t_end && c0 + (lane & 15) < t_end) my_blk = bt[(c0 + (lane & 15)) / bs];
    for (; c0 < t_end; c0 += kDecWarps * 16) {
        const int nv = min(16, t_end - c0);
        // addresses of this lane's key half-row and value pieces
        const int32_t kblk = __shfl_sync(0xffffffffu, my_blk, ktok);
        uint4 kr[HALF16];
        const bool kvalid = ktok < nv && kblk >= 0;
        if (kvalid) {
            const int32_t i = c0 + ktok;
            const T *src = kc + (int64_t)kblk * blk_stride + head_off + (int64_t)(i % bs) * D +
                           khalf * (D / 2);
#pragma unroll
            for (int p = 0; p < HALF16; ++p) kr[p] = ldg_stream(src + p * E);
        }
        uint4 vr[8];
        bool vvalid[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int t = vpar + 2 * k;
            const int32_t vb = __shfl_sync(0xffffffffu, my_blk, t);
            vvalid[k] = t < nv && vb >= 0;
            if (vvalid[k]) {
                const int32_t i = c0 + t;
                vr[k] = ldg_stream(vc + (int64_t)vb * blk_stride + head_off + (int64_t)(i % bs) * D +
                                   vpiece * E);
            }
        }
        // next chunk's block ids
        const int32_t cn = c0 + kDecWarps * 16;
        const int32_t nxt = (cn + (lane & 15) < t_end) ? bt[(cn + (lane & 15)) / bs] : -1;
        if (ktok < nv && kblk < 0 && khalf == 0) set_status(status, KVS_ERR_INVALID_ARG);

        // scores (base-2 logits) for this lane's entry
        float s[G];
#pragma unroll
        for (int g = 0; g < G; ++g) s[g] = 0.f;
        if (kvalid) {
#pragma unroll
            for (int p = 0; p < HALF16; ++p) {
                float kf[E];
                R::unpack(kr[p], kf);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float *qq = &s_q[g][khalf * (D / 2) + p * E];
#pragma unroll
                    for (int e = 0; e < E; e += 4) {
                        const float4 q4 = *reinterpret_cast<const float4 *>(qq + e);
                        s[g] = fmaf(kf[e], q4.x, s[g]);
                        s[g] = fmaf(kf[e + 1], q4.y, s[g]);
                        s[g] = fmaf(kf[e + 2], q4.z, s[g]);
                        s[g] = fmaf(kf[e + 3], q4.w, s[g]);
                    }
                }
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            s[g] += __shfl_xor_sync(0xffffffffu, s[g], 1);
            if (!kvalid) s[g] = -INFINITY;
            float cm = s[g];
#pragma unroll
            for (int off = 2; off < 32; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
            const float mn = fmaxf(m[g], cm);
            const float mref = mn == -INFINITY ? 0.f : mn;
            const float alpha = ex2(m[g] - mref);
            const float p = ex2(s[g] - mref);
            float ps = p;
#pragma unroll
            for (int off = 2; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            l[g] = l[g] * alpha + ps;
            m[g] = mn;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[g][e] *= alpha;
            if (khalf == 0) s_p[warp][ktok][g] = p;
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (!vvalid[k]) continue;
            const int t = vpar + 2 * k;
            float vf[E];
            R::unpack(vr[k], vf);
            float pp[G];
            if constexpr (G % 4 == 0) {
#pragma unroll
                for (int g = 0; g < G; g += 4) {
                    const float4 p4 = *reinterpret_cast<const float4 *>(&s_p[warp][t][g]);
                    pp[g] = p4.x; pp[g + 1] = p4.y; pp[g + 2] = p4.z; pp[g + 3] = p4.w;
                }
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g) pp[g] = s_p[warp][t][g];
            }
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < E; ++e) acc[g][e] = fmaf(pp[g], vf[e], acc[g][e]);
        }
        __syncwarp();
        my_blk = nxt;
    }
    // merge the two entry parities, then the warps
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < E; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], 16);
    if (lane < 16) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < E; ++e) s_acc[warp][g][vpiece * E + e] = acc[g][e];
    }
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            s_m[warp][g] = m[g];
            s_l[warp][g] = l[g];
        }
    }
    __syncthreads();
    const bool single = nsplit == 1;
    float *part = partials + (((int64_t)b * Hq + kvh * G) * max_splits) * (D + 2);
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, e = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, s_m[w][g]);
        const float Mr = M == -INFINITY ? 0.f : M;
        float L = 0.f, A = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float f = ex2(s_m[w][g] - Mr);
            L += s_l[w][g] * f;
            A += s_acc[w][g][e] * f;
        }
        if (single) {
            store_out(o, ((int)((int64_t)b * Hq + kvh * G + g)) * D + e, L > 0.f ? A / L : 0.f);
        } else {
            float *pp = part + ((int64_t)g * max_splits + split) * (D + 2);
            pp[e] = A;
            if (e == 0) {
                pp[D] = M;
                pp[D + 1] = L;
            }
        }
    }
}

cudaError_t launch_decode_mma(int G, const void *q, const void *kc, const void *vc,
                              const int32_t *bt, const int32_t *nt, int32_t B, int32_t Hq,
                              int32_t Hkv, int32_t bs, int32_t max_blocks, float scale_log2,
                              int32_t tps, int32_t max_splits, void *o, float *partials,
                              int32_t *status, cudaStream_t s);

// Merge the split partials of one (sequence, query head): thread e owns output
// dim e; every split's (max, sum) pair is read by all threads (broadcast).
template <typename T, int D>
__global__ void __launch_bounds__(D)
    k_decode_combine(const int32_t *__restrict__ num_tokens, int32_t Hq, int32_t bs,
                     int32_t max_blocks, int32_t tps, int32_t max_splits,
                     const float *__restrict__ partials, T *__restrict__ o) {
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
    const int32_t ntok = min(max(num_tokens[b], 0), max_blocks * bs);
    const int32_t nsplit = max(1, (ntok + tps - 1) / tps);
    if (nsplit == 1) return;  // the split kernel wrote the output itself
    const float *pg = partials + ((int64_t)b * Hq + h) * max_splits * (D + 2);
    float M = -INFINITY;
#pragma unroll 8
    for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, pg[sp * (D + 2) + D]);
    const float Mr = M == -INFINITY ? 0.f : M;
    float L = 0.f, A = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < nsplit; ++sp) {
        const float *pp = pg + sp * (D + 2);
        const float f = ex2(pp[D] - Mr);
        L += pp[D + 1] * f;
        A += pp[e] * f;
    }
    store_out(o, (int)(((int64_t)b * Hq + h) * D + e), L > 0.f ? A / L : 0.f);
}

struct DecodePlan {
    int32_t tps, max_splits;
    size_t partial_bytes;
};

// Entries per split, between 128 and 1024: the longest splits that still give
// every one of the 148 SMs a CTA when sequences are half full. Long splits keep
// each warp's copy ring busy for many chunks; shorter ones only added start-up
// and merge cost (measured on two 28 700-entry sequences with 1-token blocks:
// 1024 entries per split ran 1.7x faster than 128).
inline DecodePlan decode_plan(int32_t B, int32_t Hq, int32_t Hkv, int32_t d, int32_t bs,
                              int32_t max_blocks) {
    DecodePlan p;
    const int64_t max_tok = (int64_t)max_blocks * bs;
    const int64_t units = (int64_t)B * Hkv;
    int32_t tps = 1024;
    while (tps > 128 && units * ((max_tok / 2 + tps - 1) / tps) < 148) tps >>= 1;
    p.tps = tps;
    p.max_splits = (int32_t)std::max<int64_t>(1, (max_tok + tps - 1) / tps);
    p.partial_bytes = p.max_splits > 1 ? (size_t)B * Hq * p.max_splits * (d + 2) * sizeof(float) : 16;
    return p;
}

template <typename T, int D, int G>
void launch_decode(const void *q, const void *kc, const void *vc, const int32_t *bt,
                   const int32_t *nt, int32_t B, int32_t Hq, int32_t Hkv, int32_t bs,
                   int32_t max_blocks, float qscale, const DecodePlan &p, void *o, void *ws,
                   int32_t *status, cudaStream_t s) {
    dim3 grid(p.max_splits, Hkv, B);
    k_decode<T, D, G><<<grid, kDecWarps * 32, 0, s>>>(
        (const T *)q, (const T *)kc, (const T *)vc, bt, nt, Hq, Hkv, bs, max_blocks, qscale, p.tps,
        p.max_splits, (T *)o, (float *)ws, status);
}

}  // namespace kvs

using namespace kvs;

extern "C" size_t kvs_paged_decode_ws_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t d,
                                            int32_t block_size, int32_t max_blocks) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || block_size <= 0 || max_blocks <= 0) return 0;
    return decode_plan(B, Hq, Hkv, d, block_size, max_blocks).partial_bytes;
}

extern "C" kvs_status kvs_paged_decode_attn(const void *q, const void *k_cache, const void *v_cache,
                                            const int32_t *block_table, const int32_t *num_tokens,
                                            int32_t B, int32_t Hq, int32_t Hkv, int32_t d,
                                            int32_t block_size, int32_t max_blocks, float scale,
                                            kvs_dtype dt, void *o, void *ws, size_t ws_bytes,
                                            int32_t *dev_status, kvs_stream_t stream) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || block_size <= 0 || max_blocks <= 0)
        return KVS_ERR_INVALID_ARG;
    if (B == 0) return KVS_OK;
    if (!q || !k_cache || !v_cache || !block_table || !num_tokens || !o || !ws)
        return KVS_ERR_INVALID_ARG;
    if (((uintptr_t)q | (uintptr_t)k_cache | (uintptr_t)v_cache | (uintptr_t)ws) % 16)
        return KVS_ERR_INVALID_ARG;
    if (B > 65535 || Hkv > 65535) return KVS_ERR_CAPACITY;
    const int G = Hq / Hkv;
    const bool bf = dt == KVS_BF16 && d == 128, f32 = dt == KVS_F32 && d == 64;
    if (!bf && !f32) return KVS_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8) return KVS_ERR_UNSUPPORTED;
    const DecodePlan p = decode_plan(B, Hq, Hkv, d, block_size, max_blocks);
    if (ws_bytes < p.partial_bytes) return KVS_ERR_CAPACITY;
    const float qs = scale * 1.4426950408889634f;  // base-2 logits
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (bf) {
        // bf16: bulk-copy staging + warp-level tensor-core products
        e = launch_decode_mma(G, q, k_cache, v_cache, block_table, num_tokens, B, Hq, Hkv,
                              block_size, max_blocks, qs, p.tps, p.max_splits, o, (float *)ws,
                              dev_status, s);
        if (e != cudaSuccess) return cuda_status(e);
        if (p.max_splits > 1)
            k_decode_combine<__nv_bfloat16, 128><<<dim3(Hq, B), 128, 0, s>>>(
                num_tokens, Hq, block_size, max_blocks, p.tps, p.max_splits, (const float *)ws,
                (__nv_bfloat16 *)o);
    } else {
#define KVS_DEC(GG)                                                                              \
    launch_decode<float, 64, GG>(q, k_cache, v_cache, block_table, num_tokens, B, Hq, Hkv,       \
                                 block_size, max_blocks, qs, p, o, ws, dev_status, s)
        switch (G) {
            case 1: KVS_DEC(1); break;
            case 2: KVS_DEC(2); break;
            case 4: KVS_DEC(4); break;
            default: KVS_DEC(8); break;
        }
#undef KVS_DEC
        if (p.max_splits > 1)
            k_decode_combine<float, 64><<<dim3(Hq, B), 64, 0, s>>>(
                num_tokens, Hq, block_size, max_blocks, p.tps, p.max_splits, (const float *)ws,
                (float *)o);
    }
    return cuda_status(cudaGetLastError());
}
