// Paged decode without any device allocation by the caller or the library.
//
// Some callers cannot call cudaMalloc on their decode path: serving engines
// that replay each generation step from a captured CUDA graph, engines that
// hand all device memory to their own pool allocator and forbid allocations
// while a step runs, and embedders that only get device pointers for inputs
// and outputs. For them, kvs_paged_decode_attn_static runs the same split-K
// decode as kvs_paged_decode_attn but takes its scratch (the per-split softmax
// partials) from one fixed array compiled into this file.
//
// The array lives in device global memory of every GPU that loads this part
// of the library, for the life of the process. Its size is the stated maximum
// KVS_DECODE_STATIC_SCRATCH_BYTES; a request whose scratch would not fit is
// rejected with KVS_ERR_CAPACITY before anything is launched.
//
// In host code the array's name does not stand for a device address (it is a
// host-side shadow symbol). The device address is obtained once per device,
// with that device current, through cudaGetSymbolAddress. That set-up happens
// inside the first call on each device, so the first call must not be made
// while a stream is being captured. The address is kept together with the id
// of the CUDA context it was taken in; if the device's context has been torn
// down and rebuilt since (cudaDeviceReset), the module is loaded again and the
// array may move, so the next call looks the address up again (again not
// during a capture). Nothing in the array has to start at zero: every call
// writes the partials it later reads.
//
// All calls share the one array: two calls whose kernels overlap on the GPU
// (different streams without ordering, or concurrent host threads) race on it
// and give wrong results. Calls ordered on one stream are fine.
#include <mutex>

#include "common.cuh"

namespace kvs {

static __device__ __align__(256) unsigned char g_decode_scratch[KVS_DECODE_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void *g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Id of the calling thread's current CUDA context; 0 if there is none yet.
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked = false;
    if (!looked) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        looked = true;
    }
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array on the current device (looked up on the
// first use in each context).
kvs_status scratch_on_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return KVS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    const unsigned long long ctx = current_ctx_id();
    if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);  // makes the primary context current
        if (e != cudaSuccess) return cuda_status(e);
        if (!p) return KVS_ERR_CUDA;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = current_ctx_id();
    }
    *out = g_scratch_addr[dev];
    return KVS_OK;
}
}  // namespace

}  // namespace kvs

using namespace kvs;

extern "C" kvs_status kvs_paged_decode_attn_static(const void *q, const void *k_cache,
                                                   const void *v_cache, const int32_t *block_table,
                                                   const int32_t *num_tokens, int32_t B,
                                                   int32_t Hq, int32_t Hkv, int32_t d,
                                                   int32_t block_size, int32_t max_blocks,
                                                   int32_t pool_blocks, float scale, kvs_dtype dt,
                                                   void *o, int32_t *dev_status,
                                                   kvs_stream_t stream) {
    const size_t need = kvs_paged_decode_ws_bytes(B, Hq, Hkv, d, block_size, max_blocks);
    if (need > KVS_DECODE_STATIC_SCRATCH_BYTES) return KVS_ERR_CAPACITY;
    void *ws = nullptr;
    const kvs_status st = scratch_on_current_device(&ws);
    if (st != KVS_OK) return st;
    return kvs_paged_decode_attn(q, k_cache, v_cache, block_table, num_tokens, B, Hq, Hkv, d,
                                 block_size, max_blocks, pool_blocks, scale, dt, o, ws,
                                 KVS_DECODE_STATIC_SCRATCH_BYTES, dev_status, stream);
}
