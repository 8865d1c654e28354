// fp32 eviction-masked attention forward and backward on CUDA cores.
//
// The tensor cores have no fp32 input kind that meets a 1e-5 tolerance, so the
// fp32 path runs on FMA units. It consumes the same compiled tile mask as the
// bf16 tensor-core path: row-CSR lists for the forward and dQ, column-CSR
// lists for dK/dV; EMPTY tiles are never visited, PARTIAL tiles use the bits.
// ("KV-streams: speeding up agentic RL by operating on the KV cache directly",
// trainer replay; "KV-streams for Efficient Compaction in Agentic
// Reinforcement Learning", Fig. 2(A).)
//
// Thread layout: SPLIT = D/16 threads per row, each owning 16 consecutive
// feature dims; dot products are reduced over the SPLIT lanes. Long sums (the
// output rows, the softmax denominator, dQ, dK, dV) use compensated (Kahan)
// accumulation so fp32 rounding does not grow with the number of visible keys.
#include "common.cuh"

namespace kvs {

template <int SPLIT>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = 1; o < SPLIT; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Kahan-compensated running sum.
struct KSum {
    float s = 0.f, c = 0.f;
    __device__ __forceinline__ void add(float x) {
        const float y = x - c;
        const float t = s + y;
        c = (t - s) - y;
        s = t;
    }
    __device__ __forceinline__ void scale(float a) {
        s *= a;
        c *= a;
    }
};

constexpr int kDims = 16;  // feature dims owned by one thread

__device__ __forceinline__ bool tile_bit(const uint32_t *bits_row, int c) {
    return (bits_row[c >> 5] >> (c & 31)) & 1u;
}

// Load 128 rows x D floats of a [.., N, H, D] tensor (rows past N zeroed).
template <int D>
__device__ void load_tile(float *dst, const float *src_b, int32_t N, int32_t H, int32_t h,
                          int32_t r0) {
    for (int i = threadIdx.x; i < 128 * (D / 4); i += blockDim.x) {
        const int r = i / (D / 4), c4 = i % (D / 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r0 + r < N)
            v = *reinterpret_cast<const float4 *>(src_b + ((int64_t)(r0 + r) * H + h) * D + 4 * c4);
        *reinterpret_cast<float4 *>(dst + r * D + 4 * c4) = v;
    }
}

template <int D>
__global__ void __launch_bounds__(128 * (D / kDims), 1)
    k_fwd_simt(const float *__restrict__ q, const float *__restrict__ k,
               const float *__restrict__ v, kvs_tile_mask m, int32_t Hq, int32_t Hkv,
               float scale, float *__restrict__ o, float *__restrict__ lse) {
    constexpr int SPLIT = D / kDims;
    extern __shared__ __align__(16) float sm[];
    float *sK = sm, *sV = sm + 128 * D;
    __shared__ uint32_t sBits[128][4];
    const int qi = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int N = m.N, T = m.T, G = Hq / Hkv, kvh = h / G;
    const int r = threadIdx.x / SPLIT, part = threadIdx.x % SPLIT;
    const int t = qi * 128 + r;
    const bool live = t < N;
    float qr[kDims];
    KSum acc[kDims], l;
    const float *qrow = q + (((int64_t)b * N + (live ? t : 0)) * Hq + h) * D + part * kDims;
#pragma unroll
    for (int i = 0; i < kDims; ++i) qr[i] = live ? qrow[i] * scale : 0.f;
    float mx = -INFINITY;
    const float *kb = k + (int64_t)b * N * Hkv * D, *vb = v + (int64_t)b * N * Hkv * D;
    const int32_t e0 = m.row_ptr[b * T + qi], e1 = m.row_ptr[b * T + qi + 1];
    for (int32_t e = e0; e < e1; ++e) {
        const int32_t kj = m.row_col[e], pid = m.row_pidx[e];
        __syncthreads();
        load_tile<D>(sK, kb, N, Hkv, kvh, kj * 128);
        load_tile<D>(sV, vb, N, Hkv, kvh, kj * 128);
        if (pid >= 0)
            for (int i = threadIdx.x; i < 512; i += blockDim.x)
                sBits[i >> 2][i & 3] = m.bits[(int64_t)pid * 512 + i];
        __syncthreads();
        for (int c = 0; c < 128; ++c) {
            float s = 0.f;
            const float *kr = sK + c * D + part * kDims;
#pragma unroll
            for (int i = 0; i < kDims; ++i) s = fmaf(qr[i], kr[i], s);
            s = group_sum<SPLIT>(s);
            const bool vis = live && (pid < 0 || tile_bit(sBits[r], c));
            if (!vis) continue;
            const float *vr = sV + c * D + part * kDims;
            float p = 1.f;
            if (s > mx) {
                const float alpha = expf(mx - s);
                l.scale(alpha);
#pragma unroll
                for (int i = 0; i < kDims; ++i) acc[i].scale(alpha);
                mx = s;
            } else {
                p = expf(s - mx);
            }
            l.add(p);
#pragma unroll
            for (int i = 0; i < kDims; ++i) acc[i].add(p * vr[i]);
        }
    }
    if (!live) return;
    const float lsum = l.s;
    float *orow = o + (((int64_t)b * N + t) * Hq + h) * D + part * kDims;
#pragma unroll
    for (int i = 0; i < kDims; ++i) orow[i] = lsum > 0.f ? acc[i].s / lsum : 0.f;
    if (part == 0) lse[((int64_t)b * Hq + h) * N + t] = lsum > 0.f ? mx + logf(lsum) : -INFINITY;
}

// D_t = <dO_t, O_t> (fp32), one warp per row.
__global__ void k_rowdot_f32(const float *__restrict__ o, const float *__restrict__ dO,
                             int64_t rows, int32_t D, float *__restrict__ out_d, int32_t N,
                             int32_t Hq) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float s = 0.f;
    for (int i = lane; i < D; i += 32) s = fmaf(o[row * D + i], dO[row * D + i], s);
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    // row = (b*N + t)*Hq + h  ->  out_d[(b*Hq + h)*N + t]
    if (lane == 0) {
        const int64_t h = row % Hq, bt = row / Hq, t = bt % N, b = bt / N;
        out_d[(b * Hq + h) * N + t] = s;
    }
}

template <int D>
__global__ void __launch_bounds__(128 * (D / kDims), 1)
    k_dq_simt(const float *__restrict__ q, const float *__restrict__ k,
              const float *__restrict__ v, const float *__restrict__ dO,
              const float *__restrict__ lse, const float *__restrict__ Drow, kvs_tile_mask m,
              int32_t Hq, int32_t Hkv, float scale, float *__restrict__ dq) {
    constexpr int SPLIT = D / kDims;
    extern __shared__ __align__(16) float sm[];
    float *sK = sm, *sV = sm + 128 * D;
    __shared__ uint32_t sBits[128][4];
    const int qi = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int N = m.N, T = m.T, G = Hq / Hkv, kvh = h / G;
    const int r = threadIdx.x / SPLIT, part = threadIdx.x % SPLIT;
    const int t = qi * 128 + r;
    const bool live = t < N;
    float qr[kDims], dor[kDims];
    KSum acc[kDims];
    const int64_t rowoff = (((int64_t)b * N + (live ? t : 0)) * Hq + h) * D + part * kDims;
#pragma unroll
    for (int i = 0; i < kDims; ++i) {
        qr[i] = live ? q[rowoff + i] : 0.f;
        dor[i] = live ? dO[rowoff + i] : 0.f;
    }
    const float L = live ? lse[((int64_t)b * Hq + h) * N + t] : 0.f;
    const float Dt = live ? Drow[((int64_t)b * Hq + h) * N + t] : 0.f;
    const float *kb = k + (int64_t)b * N * Hkv * D, *vb = v + (int64_t)b * N * Hkv * D;
    const int32_t e0 = m.row_ptr[b * T + qi], e1 = m.row_ptr[b * T + qi + 1];
    for (int32_t e = e0; e < e1; ++e) {
        const int32_t kj = m.row_col[e], pid = m.row_pidx[e];
        __syncthreads();
        load_tile<D>(sK, kb, N, Hkv, kvh, kj * 128);
        load_tile<D>(sV, vb, N, Hkv, kvh, kj * 128);
        if (pid >= 0)
            for (int i = threadIdx.x; i < 512; i += blockDim.x)
                sBits[i >> 2][i & 3] = m.bits[(int64_t)pid * 512 + i];
        __syncthreads();
        for (int c = 0; c < 128; ++c) {
            const float *kr = sK + c * D + part * kDims, *vr = sV + c * D + part * kDims;
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int i = 0; i < kDims; ++i) {
                s = fmaf(qr[i], kr[i], s);
                dp = fmaf(dor[i], vr[i], dp);
            }
            s = group_sum<SPLIT>(s);
            dp = group_sum<SPLIT>(dp);
            const bool vis = live && (pid < 0 || tile_bit(sBits[r], c));
            if (!vis) continue;
            const float p = expf(s * scale - L);
            const float ds = p * (dp - Dt);
#pragma unroll
            for (int i = 0; i < kDims; ++i) acc[i].add(ds * kr[i]);
        }
    }
    if (!live) return;
    float *out = dq + rowoff;
#pragma unroll
    for (int i = 0; i < kDims; ++i) out[i] = acc[i].s * scale;
}

template <int D>
__global__ void __launch_bounds__(128 * (D / kDims), 1)
    k_dkdv_simt(const float *__restrict__ q, const float *__restrict__ k,
                const float *__restrict__ v, const float *__restrict__ dO,
                const float *__restrict__ lse, const float *__restrict__ Drow, kvs_tile_mask m,
                int32_t Hq, int32_t Hkv, float scale, float *__restrict__ dk,
                float *__restrict__ dv) {
    constexpr int SPLIT = D / kDims;
    extern __shared__ __align__(16) float sm[];
    float *sQ = sm, *sO = sm + 128 * D;
    __shared__ uint32_t sBits[128][4];
    __shared__ float sL[128], sD[128];
    const int kj = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int N = m.N, T = m.T, G = Hq / Hkv;
    const int c = threadIdx.x / SPLIT, part = threadIdx.x % SPLIT;
    const int j = kj * 128 + c;
    const bool live = j < N;
    float kr[kDims], vr[kDims];
    KSum adk[kDims], adv[kDims];
    const int64_t rowoff = (((int64_t)b * N + (live ? j : 0)) * Hkv + kvh) * D + part * kDims;
#pragma unroll
    for (int i = 0; i < kDims; ++i) {
        kr[i] = live ? k[rowoff + i] : 0.f;
        vr[i] = live ? v[rowoff + i] : 0.f;
    }
    const float *qb = q + (int64_t)b * N * Hq * D, *ob = dO + (int64_t)b * N * Hq * D;
    const int32_t e0 = m.col_ptr[b * T + kj], e1 = m.col_ptr[b * T + kj + 1];
    for (int g = 0; g < G; ++g) {
        const int h = kvh * G + g;
        for (int32_t e = e0; e < e1; ++e) {
            const int32_t qi = m.col_row[e], pid = m.col_pidx[e];
            __syncthreads();
            load_tile<D>(sQ, qb, N, Hq, h, qi * 128);
            load_tile<D>(sO, ob, N, Hq, h, qi * 128);
            for (int i = threadIdx.x; i < 128; i += blockDim.x) {
                const int t = qi * 128 + i;
                sL[i] = t < N ? lse[((int64_t)b * Hq + h) * N + t] : 0.f;
                sD[i] = t < N ? Drow[((int64_t)b * Hq + h) * N + t] : 0.f;
            }
            if (pid >= 0)
                for (int i = threadIdx.x; i < 512; i += blockDim.x)
                    sBits[i >> 2][i & 3] = m.bits[(int64_t)pid * 512 + i];
            __syncthreads();
            for (int r = 0; r < 128; ++r) {
                const float *qr = sQ + r * D + part * kDims, *dr = sO + r * D + part * kDims;
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int i = 0; i < kDims; ++i) {
                    s = fmaf(qr[i], kr[i], s);
                    dp = fmaf(dr[i], vr[i], dp);
                }
                s = group_sum<SPLIT>(s);
                dp = group_sum<SPLIT>(dp);
                const bool vis = live && (pid < 0 || tile_bit(sBits[r], c));
                if (!vis) continue;
                const float p = expf(s * scale - sL[r]);
                const float ds = p * (dp - sD[r]);
#pragma unroll
                for (int i = 0; i < kDims; ++i) {
                    adv[i].add(p * dr[i]);
                    adk[i].add(ds * qr[i]);
                }
            }
        }
    }
    if (!live) return;
#pragma unroll
    for (int i = 0; i < kDims; ++i) {
        dk[rowoff + i] = adk[i].s * scale;
        dv[rowoff + i] = adv[i].s;
    }
}

template <int D>
static cudaError_t fwd_simt(const float *q, const float *k, const float *v, const kvs_tile_mask &m,
                            int32_t Hq, int32_t Hkv, float scale, float *o, float *lse,
                            cudaStream_t s) {
    const size_t smem = 2 * 128 * D * sizeof(float);
    cudaFuncSetAttribute(k_fwd_simt<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid(m.T, Hq, m.B);
    k_fwd_simt<D><<<grid, 128 * (D / kDims), smem, s>>>(q, k, v, m, Hq, Hkv, scale, o, lse);
    return cudaGetLastError();
}

template <int D>
static cudaError_t bwd_simt(const float *q, const float *k, const float *v, const float *o,
                            const float *dO, const float *lse, const kvs_tile_mask &m, int32_t Hq,
                            int32_t Hkv, float scale, float *dq, float *dk, float *dv,
                            float *Drow, cudaStream_t s) {
    const int64_t rows = (int64_t)m.B * m.N * Hq;
    k_rowdot_f32<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(o, dO, rows, D, Drow, m.N, Hq);
    const size_t smem = 2 * 128 * D * sizeof(float);
    cudaFuncSetAttribute(k_dq_simt<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_dkdv_simt<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_dq_simt<D><<<dim3(m.T, Hq, m.B), 128 * (D / kDims), smem, s>>>(q, k, v, dO, lse, Drow, m, Hq,
                                                                 Hkv, scale, dq);
    k_dkdv_simt<D><<<dim3(m.T, Hkv, m.B), 128 * (D / kDims), smem, s>>>(q, k, v, dO, lse, Drow, m, Hq,
                                                                    Hkv, scale, dk, dv);
    return cudaGetLastError();
}

cudaError_t launch_fwd_simt(const float *q, const float *k, const float *v, const kvs_tile_mask &m,
                            int32_t Hq, int32_t Hkv, int32_t d, float scale, float *o, float *lse,
                            cudaStream_t s) {
    return d == 64 ? fwd_simt<64>(q, k, v, m, Hq, Hkv, scale, o, lse, s)
                   : fwd_simt<128>(q, k, v, m, Hq, Hkv, scale, o, lse, s);
}

cudaError_t launch_bwd_simt(const float *q, const float *k, const float *v, const float *o,
                            const float *dO, const float *lse, const kvs_tile_mask &m, int32_t Hq,
                            int32_t Hkv, int32_t d, float scale, float *dq, float *dk, float *dv,
                            float *Drow, cudaStream_t s) {
    return d == 64 ? bwd_simt<64>(q, k, v, o, dO, lse, m, Hq, Hkv, scale, dq, dk, dv, Drow, s)
                   : bwd_simt<128>(q, k, v, o, dO, lse, m, Hq, Hkv, scale, dq, dk, dv, Drow, s);
}

}  // namespace kvs
