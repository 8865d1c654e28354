// Split-K paged decode over a compacted block table.
//
// "KV-streams: speeding up agentic RL by operating on the KV cache directly":
// generation continues from the cache entries that survived compaction; the
// cache is paged (16-token blocks, or 1-token blocks) and found through a
// block table without holes, which the attention walks in order.
//
// The CTAs share the step's live entries equally (decode_sched.cuh). For each
// piece (a contiguous range of live entries of one sequence and kv head) a CTA
// serves all G = Hq/Hkv query heads of the kv head (each K/V byte is read from
// HBM once). Each warp takes 16-entry chunks: lanes (2 per entry) dot 128-byte
// halves of the key rows with the queries held in shared memory, the warp runs
// an online softmax (base-2, pre-scaled logits), and lanes (16 per row, 2 rows
// at a time) accumulate 16-byte slices of the value rows. Warp states merge in
// shared memory; a piece that is a whole unit writes the output, any other its
// partial, and k_decode_combine folds the partials of each unit.
#include <algorithm>

#include "decode_sched.cuh"

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

__device__ __forceinline__ void store_out(float *o, int64_t i, float v) { o[i] = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *o, int64_t i, float v) {
    o[i] = __float2bfloat16_rn(v);
}

// partials: slot c + u holds G rows of D + 2 fp32 (unnormalised output, max, sum)
template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecThreads)
    k_decode(const T *__restrict__ q, const T *__restrict__ kc, const T *__restrict__ vc,
             const int32_t *__restrict__ block_table, const int32_t *__restrict__ num_tokens,
             int32_t B, int32_t Hq, int32_t Hkv, int32_t bs, int32_t max_blocks,
             int32_t pool_blocks, float qscale, int64_t n_cta, int64_t *pre_ws, float *partials,
             T *__restrict__ o, int32_t *status) {
    using R = Row16<T>;
    constexpr int E = R::E;           // elements per 16 bytes
    static_assert(D * sizeof(T) == 256, "rows are 256 bytes");
    static_assert(kDecWarps * 32 == kDecThreads, "decode work split");
    constexpr int HALF16 = 8;         // 16-byte pieces per half row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // max_blocks * bs fits in int32 (checked by the host); counts outside
    // [0, max_blocks * bs] are reported (by CTA 0) and clamped
    const int32_t cap = max_blocks * bs;
    const DecodeRange rg = dec_locate(num_tokens, B, Hkv, cap, n_cta, pre_ws, status);
    if (rg.x0 >= rg.x1) return;

    __shared__ __align__(16) float s_q[G][D];
    __shared__ __align__(16) float s_p[kDecWarps][16][G];
    __shared__ float s_m[kDecWarps][G], s_l[kDecWarps][G];
    __shared__ __align__(16) float s_acc[kDecWarps][G][D];

    const int64_t blk_stride = (int64_t)Hkv * bs * D;
    const int ktok = lane >> 1, khalf = lane & 1;    // key phase: entry, half row
    const int vpiece = lane & 15, vpar = lane >> 4;  // value phase: 16-B piece, entry parity
    int32_t b = rg.b0;
    int32_t pre = rg.pre_b0;
    int32_t ntok = dec_ntok(num_tokens, b, cap);
    int32_t nch = dec_nch(ntok);
    int32_t kvh = (rg.x0 - Hkv * pre) / nch;
    for (;;) {
        const int32_t cs = Hkv * pre + kvh * nch, ce = cs + nch;
        const int32_t ps = max(rg.x0, cs), pe = min(rg.x1, ce);
        const int32_t t_begin = (ps - cs) * kDecChunk;
        const int32_t t_end = min(ntok, (pe - cs) * kDecChunk);
        const bool whole = ps == cs && pe == ce;
        for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
            const int g = i / D, e = i % D;
            s_q[g][e] = (float)q[((int64_t)b * Hq + kvh * G + g) * D + e] * qscale;
        }
        __syncthreads();
        const int32_t *bt = block_table + (int64_t)b * max_blocks;
        const int64_t head_off = (int64_t)kvh * bs * D;

        float m[G], l[G], acc[G][E];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[g][e] = 0.f;
        }
        int32_t c0 = t_begin + warp * 16;
        int32_t my_blk = -1;
        if (c0 < t_end && c0 + (lane & 15) < t_end) my_blk = bt[(c0 + (lane & 15)) / bs];
        for (; c0 < t_end; c0 += kDecWarps * 16) {
            const int nv = min(16, t_end - c0);
            // addresses of this lane's key half-row and value pieces
            const int32_t kblk = __shfl_sync(0xffffffffu, my_blk, ktok);
            uint4 kr[HALF16];
            const bool kvalid = ktok < nv && kblk >= 0 && kblk < pool_blocks;
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
                vvalid[k] = t < nv && vb >= 0 && vb < pool_blocks;
                if (vvalid[k]) {
                    const int32_t i = c0 + t;
                    vr[k] = ldg_stream(vc + (int64_t)vb * blk_stride + head_off + (int64_t)(i % bs) * D +
                                       vpiece * E);
                }
            }
            // next chunk's block ids
            const int32_t cn = c0 + kDecWarps * 16;
            const int32_t nxt = (cn + (lane & 15) < t_end) ? bt[(cn + (lane & 15)) / bs] : -1;
            if (ktok < nv && (kblk < 0 || kblk >= pool_blocks) && khalf == 0)
                set_status(status, KVS_ERR_INVALID_ARG);

            // scores (base-2 logits) for this lane's entry
            float sc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) sc[g] = 0.f;
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
                            sc[g] = fmaf(kf[e], q4.x, sc[g]);
                            sc[g] = fmaf(kf[e + 1], q4.y, sc[g]);
                            sc[g] = fmaf(kf[e + 2], q4.z, sc[g]);
                            sc[g] = fmaf(kf[e + 3], q4.w, sc[g]);
                        }
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], 1);
                if (!kvalid) sc[g] = -INFINITY;
                float cm = sc[g];
#pragma unroll
                for (int off = 2; off < 32; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
                const float mn = fmaxf(m[g], cm);
                const float mref = mn == -INFINITY ? 0.f : mn;
                const float alpha = ex2(m[g] - mref);
                const float p = ex2(sc[g] - mref);
                float ps2 = p;
#pragma unroll
                for (int off = 2; off < 32; off <<= 1) ps2 += __shfl_xor_sync(0xffffffffu, ps2, off);
                l[g] = l[g] * alpha + ps2;
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
        const int64_t u = (int64_t)b * Hkv + kvh;
        float *part = partials + (((int64_t)blockIdx.x + u) * G) * (D + 2);  // slot c + u
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
            if (whole) {
                store_out(o, ((int64_t)b * Hq + kvh * G + g) * D + e, L > 0.f ? A / L : 0.f);
            } else {
                float *pp = part + (int64_t)g * (D + 2);
                pp[e] = A;
                if (e == 0) {
                    pp[D] = M;
                    pp[D + 1] = L;
                }
            }
        }
        if (pe >= rg.x1) break;
        __syncthreads();  // s_q, s_acc, s_m, s_l are rewritten for the next piece
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

cudaError_t launch_decode_mma(int G, const void *q, const void *kc, const void *vc,
                              const int32_t *bt, const int32_t *nt, int32_t B, int32_t Hq,
                              int32_t Hkv, int32_t bs, int32_t max_blocks, int32_t pool_blocks,
                              float scale_log2, int64_t n_cta, int64_t *pre_ws, float *partials,
                              void *o, int32_t *status, cudaStream_t s);

// Merge the partials of one (sequence, query head): thread e owns output dim e.
// The unit's pieces sit in the CTAs of its first and last chunk and the ones
// between; a unit held by one CTA was written by it directly, one without live
// entries gets zeros. The pieces' maxima and sums are read by the block in
// parallel (one piece per thread) and reduced; each piece's weight 2^(m - M)
// goes to shared memory, and every thread then sums its dimension over the
// pieces with independent loads.
template <int D>
__device__ __forceinline__ float block_reduce(float v, bool is_max, float *s_red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float w = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmaxf(v, w) : v + w;
    }
    __syncthreads();  // s_red is free (a previous reduction has been read)
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = s_red[0];
#pragma unroll
    for (int w = 1; w < D / 32; ++w) r = is_max ? fmaxf(r, s_red[w]) : r + s_red[w];
    return r;
}

template <typename T, int D>
__global__ void __launch_bounds__(D)
    k_decode_combine(const int32_t *__restrict__ num_tokens, int32_t B, int32_t Hq, int32_t Hkv,
                     int32_t cap, int64_t n_cta, const int64_t *__restrict__ pre_ws,
                     const float *__restrict__ partials, T *__restrict__ o) {
    static_assert(D % 32 == 0 && D >= 32, "whole warps");
    __shared__ float s_w[kDecWave];  // weight of each piece (at most one per CTA)
    __shared__ float s_red[D / 32];
    const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
    const int G = Hq / Hkv, kvh = h / G, g = h % G;
    const int64_t nch = dec_nch(dec_ntok(num_tokens, b, cap));
    const int64_t oi = ((int64_t)b * Hq + h) * D + e;
    if (nch == 0) {
        store_out(o, oi, 0.f);
        return;
    }
    const int64_t tc = (int64_t)Hkv * pre_ws[B];
    const int64_t cs = (int64_t)Hkv * pre_ws[b] + (int64_t)kvh * nch;
    const int64_t c_first = dec_cta_of(cs, tc, n_cta), c_last = dec_cta_of(cs + nch - 1, tc, n_cta);
    if (c_first == c_last) return;  // one piece: written by its CTA
    const int64_t u = (int64_t)b * Hkv + kvh;
    // With at least as many chunks as CTAs every CTA in [c_first, c_last] holds a
    // piece of the unit. With fewer, each CTA holds at most one chunk, and the
    // unit's pieces are the CTAs of its chunks. Either way there are at most
    // n_cta <= kDecWave pieces.
    const bool per_chunk = tc < n_cta;
    const int n_it = (int)(per_chunk ? nch : c_last - c_first + 1);
    auto row = [&](int i) {
        const int64_t slot = (per_chunk ? dec_cta_of(cs + i, tc, n_cta) : c_first + i) + u;
        return partials + (slot * G + g) * (D + 2);
    };
    // this thread's dimension of the first pieces, loaded before (and so overlapping)
    // the two reductions that give the pieces' weights
    constexpr int kPf = 32;
    float pv[kPf];
#pragma unroll
    for (int i = 0; i < kPf; ++i) pv[i] = i < n_it ? row(i)[e] : 0.f;
    float mloc = -INFINITY;
    for (int i = e; i < n_it; i += D) mloc = fmaxf(mloc, row(i)[D]);
    const float M = block_reduce<D>(mloc, true, s_red);
    const float Mr = M == -INFINITY ? 0.f : M;
    float lloc = 0.f;
    for (int i = e; i < n_it; i += D) {
        const float *pp = row(i);
        const float f = ex2(pp[D] - Mr);
        s_w[i] = f;
        lloc += pp[D + 1] * f;
    }
    const float L = block_reduce<D>(lloc, false, s_red);  // its barriers also publish s_w
    float A = 0.f;
#pragma unroll
    for (int i = 0; i < kPf; ++i)
        if (i < n_it) A += pv[i] * s_w[i];
#pragma unroll 8
    for (int i = kPf; i < n_it; ++i) A += row(i)[e] * s_w[i];
    store_out(o, oi, L > 0.f ? A / L : 0.f);
}

template <typename T, int D, int G>
void launch_decode(const void *q, const void *kc, const void *vc, const int32_t *bt,
                   const int32_t *nt, int32_t B, int32_t Hq, int32_t Hkv, int32_t bs,
                   int32_t max_blocks, int32_t pool_blocks, float qscale, const DecodePlan &p,
                   int64_t *pre_ws, float *partials, void *o, int32_t *status, cudaStream_t s) {
    k_decode<T, D, G><<<(unsigned)p.ctas, kDecThreads, 0, s>>>(
        (const T *)q, (const T *)kc, (const T *)vc, bt, nt, B, Hq, Hkv, bs, max_blocks, pool_blocks,
        qscale, p.ctas, pre_ws, partials, (T *)o, status);
}

}  // namespace kvs

using namespace kvs;

extern "C" size_t kvs_paged_decode_ws_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t d,
                                            int32_t block_size, int32_t max_blocks) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || block_size <= 0 || max_blocks <= 0 || Hq % Hkv)
        return 0;
    return decode_plan(B, Hq, Hkv, d, block_size, max_blocks).ws_bytes;
}

extern "C" kvs_status kvs_paged_decode_attn(const void *q, const void *k_cache, const void *v_cache,
                                            const int32_t *block_table, const int32_t *num_tokens,
                                            int32_t B, int32_t Hq, int32_t Hkv, int32_t d,
                                            int32_t block_size, int32_t max_blocks,
                                            int32_t pool_blocks, float scale, kvs_dtype dt,
                                            void *o, void *ws, size_t ws_bytes,
                                            int32_t *dev_status, kvs_stream_t stream) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || block_size <= 0 || max_blocks <= 0 ||
        pool_blocks <= 0)
        return KVS_ERR_INVALID_ARG;
    if ((int64_t)max_blocks * block_size > INT32_MAX) return KVS_ERR_CAPACITY;
    if (B == 0) return KVS_OK;
    if (!q || !k_cache || !v_cache || !block_table || !num_tokens || !o || !ws)
        return KVS_ERR_INVALID_ARG;
    if (((uintptr_t)q | (uintptr_t)k_cache | (uintptr_t)v_cache | (uintptr_t)ws) % 16)
        return KVS_ERR_INVALID_ARG;
    if (B > 65535) return KVS_ERR_CAPACITY;
    const int G = Hq / Hkv;
    const bool bf = dt == KVS_BF16 && d == 128, f32 = dt == KVS_F32 && d == 64;
    if (!bf && !f32) return KVS_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8) return KVS_ERR_UNSUPPORTED;
    const DecodePlan p = decode_plan(B, Hq, Hkv, d, block_size, max_blocks);
    if (ws_bytes < p.ws_bytes) return KVS_ERR_CAPACITY;
    // chunk coordinates are 32-bit on the device
    if (p.units * (((int64_t)max_blocks * block_size + kDecChunk - 1) / kDecChunk) > INT32_MAX)
        return KVS_ERR_CAPACITY;
    int64_t *pre = reinterpret_cast<int64_t *>(static_cast<char *>(ws) + p.pre_off);
    float *part = reinterpret_cast<float *>(static_cast<char *>(ws) + p.part_off);
    const float qs = scale * 1.4426950408889634f;  // base-2 logits
    const int32_t cap = max_blocks * block_size;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (bf) {
        // bf16: cp.async staging + warp-level tensor-core products
        e = launch_decode_mma(G, q, k_cache, v_cache, block_table, num_tokens, B, Hq, Hkv,
                              block_size, max_blocks, pool_blocks, qs, p.ctas, pre, part, o,
                              dev_status, s);
        if (e != cudaSuccess) return cuda_status(e);
        k_decode_combine<__nv_bfloat16, 128><<<dim3(Hq, B), 128, 0, s>>>(
            num_tokens, B, Hq, Hkv, cap, p.ctas, pre, part, (__nv_bfloat16 *)o);
    } else {
#define KVS_DEC(GG)                                                                              \
    launch_decode<float, 64, GG>(q, k_cache, v_cache, block_table, num_tokens, B, Hq, Hkv,       \
                                 block_size, max_blocks, pool_blocks, qs, p, pre, part, o,       \
                                 dev_status, s)
        switch (G) {
            case 1: KVS_DEC(1); break;
            case 2: KVS_DEC(2); break;
            case 4: KVS_DEC(4); break;
            default: KVS_DEC(8); break;
        }
#undef KVS_DEC
        k_decode_combine<float, 64><<<dim3(Hq, B), 64, 0, s>>>(num_tokens, B, Hq, Hkv, cap, p.ctas, pre,
                                                               part, (float *)o);
    }
    return cuda_status(cudaGetLastError());
}
