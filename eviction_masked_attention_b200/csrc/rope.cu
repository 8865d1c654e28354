// Rotary embedding at logical positions, with an optional scatter of the
// rotated keys (and unrotated values) into paged cache slots.
//
// "KV-streams: speeding up agentic RL by operating on the KV cache directly",
// first fix: a key keeps the rotation of its original position even after it
// moves to another physical slot, and new queries/keys continue the original
// position count -- so the position is a logical one, stored apart from the
// slot.
//
// Rotate-half pairs (i, i + d/2) with angle p * theta^(-2i/d). The angle is
// formed and reduced modulo 2*pi in fp64 (positions reach 2^17 and more), the
// rotation itself runs in fp32.
#include "common.cuh"

namespace kvs {

template <typename T>
struct Vec4;  // 4 consecutive elements
template <>
struct Vec4<float> {
    using raw = float4;
    __device__ static void unpack(raw r, float (&f)[4]) { f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w; }
    __device__ static raw pack(const float (&f)[4]) { return make_float4(f[0], f[1], f[2], f[3]); }
};
template <>
struct Vec4<__nv_bfloat16> {
    using raw = uint2;
    __device__ static void unpack(raw r, float (&f)[4]) {
        f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x); f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
    }
    __device__ static raw pack(const float (&f)[4]) {
        return make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
    }
};

// One CTA per token; thread t handles pairs i = 4*(t % (D/8)) .. +3 of head
// group t / (D/8), looping over heads.
template <typename T, int D>
__global__ void k_rope(const T *__restrict__ x, int64_t x_stride, T *__restrict__ y,
                       const int32_t *__restrict__ lpos, int32_t n_tok, int32_t H, double log2_theta,
                       int32_t inverse, const int64_t *__restrict__ out_slot, int32_t bs,
                       int64_t n_slots, const T *__restrict__ v, int64_t v_stride,
                       T *__restrict__ v_out, int32_t *status) {
    constexpr int kThreadsPerHead = D / 8;  // each thread: 4 pairs
    const int32_t n = blockIdx.x;
    if (n >= n_tok) return;
    const int sub = threadIdx.x % kThreadsPerHead;
    const int hstep = blockDim.x / kThreadsPerHead;
    const int i0 = 4 * sub;
    double p = (double)lpos[n];
    if (inverse) p = -p;
    float c[4], s[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const double inv_freq = exp2(-(2.0 * (i0 + k) / D) * log2_theta);
        const double ang = p * inv_freq;
        const double twopi = 6.283185307179586476925286766559;
        const double red = ang - twopi * rint(ang / twopi);
        sincosf((float)red, &s[k], &c[k]);
    }
    int64_t orow = 0;
    bool to_cache = out_slot != nullptr;
    if (to_cache) {
        const int64_t slot = out_slot[n];
        if (slot < 0 || slot >= n_slots) {  // outside the cache: reported, row skipped
            if (threadIdx.x == 0) set_status(status, KVS_ERR_INVALID_ARG);
            return;
        }
        orow = (slot / bs) * (int64_t)H * bs * D + (slot % bs) * D;  // + h*bs*D
    }
    using V4 = Vec4<T>;
    for (int h = threadIdx.x / kThreadsPerHead; h < H; h += hstep) {
        const T *xr = x + (int64_t)n * x_stride + (int64_t)h * D;
        float a[4], b[4], ya[4], yb[4];
        V4::unpack(*reinterpret_cast<const typename V4::raw *>(xr + i0), a);
        V4::unpack(*reinterpret_cast<const typename V4::raw *>(xr + i0 + D / 2), b);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            ya[k] = a[k] * c[k] - b[k] * s[k];
            yb[k] = a[k] * s[k] + b[k] * c[k];
        }
        T *yr = to_cache ? y + orow + (int64_t)h * bs * D : y + ((int64_t)n * H + h) * D;
        *reinterpret_cast<typename V4::raw *>(yr + i0) = V4::pack(ya);
        *reinterpret_cast<typename V4::raw *>(yr + i0 + D / 2) = V4::pack(yb);
        if (to_cache && v) {
            const T *vr = v + (int64_t)n * v_stride + (int64_t)h * D;
            T *vo = v_out + orow + (int64_t)h * bs * D;
            *reinterpret_cast<typename V4::raw *>(vo + i0) =
                *reinterpret_cast<const typename V4::raw *>(vr + i0);
            *reinterpret_cast<typename V4::raw *>(vo + i0 + D / 2) =
                *reinterpret_cast<const typename V4::raw *>(vr + i0 + D / 2);
        }
    }
}

}  // namespace kvs

using namespace kvs;

extern "C" kvs_status kvs_rope_logical(const void *x, int64_t x_tok_stride, void *y,
                                       const int32_t *lpos, int32_t n_tok, int32_t H, int32_t d,
                                       double theta, int32_t inverse, const int64_t *out_slot,
                                       int32_t block_size, int32_t pool_blocks, const void *v,
                                       int64_t v_tok_stride, void *v_out, kvs_dtype dt,
                                       int32_t *dev_status, kvs_stream_t stream) {
    if (n_tok < 0 || H <= 0 || !(theta > 1.0)) return KVS_ERR_INVALID_ARG;
    if (n_tok == 0) return KVS_OK;
    if (!x || !y || !lpos) return KVS_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return KVS_ERR_UNSUPPORTED;
    if (dt != KVS_F32 && dt != KVS_BF16) return KVS_ERR_UNSUPPORTED;
    if (x_tok_stride < (int64_t)H * d) return KVS_ERR_INVALID_ARG;
    const int esz = dt == KVS_F32 ? 4 : 2;
    // vector accesses: 8 bytes (bf16) / 16 bytes (fp32) per thread
    const uintptr_t need = dt == KVS_F32 ? 16 : 8;
    if (((uintptr_t)x | (uintptr_t)y) % need || (x_tok_stride * esz) % need) return KVS_ERR_INVALID_ARG;
    int64_t n_slots = 0;
    if (out_slot) {
        if (block_size <= 0 || pool_blocks <= 0) return KVS_ERR_INVALID_ARG;
        n_slots = (int64_t)pool_blocks * block_size;
        if (v) {
            if (!v_out || v_tok_stride < (int64_t)H * d) return KVS_ERR_INVALID_ARG;
            if (((uintptr_t)v | (uintptr_t)v_out) % need || (v_tok_stride * esz) % need)
                return KVS_ERR_INVALID_ARG;
        }
    } else {
        v = nullptr;
        v_out = nullptr;
        block_size = 1;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const double l2t = log2(theta);
    const int threads = 128;
    if (dt == KVS_F32) {
        if (d == 64)
            k_rope<float, 64><<<n_tok, threads, 0, s>>>((const float *)x, x_tok_stride, (float *)y,
                                                        lpos, n_tok, H, l2t, inverse, out_slot,
                                                        block_size, n_slots, (const float *)v, v_tok_stride,
                                                        (float *)v_out, dev_status);
        else
            k_rope<float, 128><<<n_tok, threads, 0, s>>>((const float *)x, x_tok_stride, (float *)y,
                                                         lpos, n_tok, H, l2t, inverse, out_slot,
                                                         block_size, n_slots, (const float *)v, v_tok_stride,
                                                         (float *)v_out, dev_status);
    } else {
        using bf = __nv_bfloat16;
        if (d == 64)
            k_rope<bf, 64><<<n_tok, threads, 0, s>>>((const bf *)x, x_tok_stride, (bf *)y, lpos,
                                                     n_tok, H, l2t, inverse, out_slot, block_size,
                                                     n_slots, (const bf *)v, v_tok_stride, (bf *)v_out,
                                                     dev_status);
        else
            k_rope<bf, 128><<<n_tok, threads, 0, s>>>((const bf *)x, x_tok_stride, (bf *)y, lpos,
                                                      n_tok, H, l2t, inverse, out_slot, block_size,
                                                      n_slots, (const bf *)v, v_tok_stride, (bf *)v_out,
                                                      dev_status);
    }
    return cuda_status(cudaGetLastError());
}
