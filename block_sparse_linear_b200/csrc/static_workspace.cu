// spla_decode_static_workspace: spla_decode with library-owned scratch.
//
// Some callers cannot allocate device memory at the point where they decode: a
// plain C host program that embeds this library without a device allocator of
// its own, or a serving engine that handed all free HBM to its KV-cache pool at
// start-up and has no room left to carve a per-call workspace from. For them the
// decode scratch lives in one file-scope __device__ array, sized at build time,
// and this entry point allocates nothing (no cudaMalloc, no cudaFree, no
// allocating library routine).
//
// The array is shared by every call on a device. Nothing in it has to start at
// zero: each decode kernel writes every word of scratch it owns before a later
// kernel of the same call reads it, so no clearing is needed or done. Two calls
// whose kernels overlap on the GPU (on different streams without ordering
// between them) use the same words and race.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace spla {
void set_last_cuda_error(int32_t e);
}

namespace {

constexpr int kMaxDevices = 64;

static_assert(SPLA_STATIC_WORKSPACE_BYTES % 256 == 0, "static workspace must be 256-byte granular");

__device__ __align__(256) unsigned char g_static_ws[SPLA_STATIC_WORKSPACE_BYTES];

std::mutex g_setup_mutex;
void* g_static_ws_ptr[kMaxDevices] = {};
unsigned long long g_static_ws_ctx[kMaxDevices] = {};   // context the pointer belongs to

// Unique id (for the life of the process) of the calling thread's current context,
// through the driver entry points the runtime exposes; false when there is none.
bool current_context_id(unsigned long long* id) {
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_static_ws on device `dev`, which must be current. It is looked
// up on the first call and again whenever the device's context has changed since
// (a cudaDeviceReset reloads the module, and the array may move), or on every call
// when the context cannot be identified.
spla_status static_ws_for(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    unsigned long long id = 0;
    const bool known = current_context_id(&id);
    if (!g_static_ws_ptr[dev] || !known || id != g_static_ws_ctx[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess) {
            spla::set_last_cuda_error((int32_t)e);
            return SPLA_ERR_CUDA;
        }
        // the lookup made the device's context current if it was not yet
        const bool now_known = current_context_id(&id);
        g_static_ws_ptr[dev] = now_known ? p : nullptr;
        g_static_ws_ctx[dev] = now_known ? id : 0;
        *out = p;
        return SPLA_OK;
    }
    *out = g_static_ws_ptr[dev];
    return SPLA_OK;
}

}  // namespace

extern "C" spla_status spla_decode_static_workspace(const spla_params* params,
                                                    const spla_cache* cache, const void* q,
                                                    const float* rms_gamma, void* out,
                                                    int32_t* sel_idx, float* o_sparse_dbg,
                                                    float* o_rla_dbg, int32_t* dev_status,
                                                    void* stream) {
    if (!cache) return SPLA_ERR_INVALID_ARG;
    // The size check runs on the host before any CUDA call.
    size_t need = 0;
    spla_status st = spla_decode_workspace_size(params, cache->batch, cache->max_blocks_per_seq,
                                                &need);
    if (st != SPLA_OK) return st;
    if (need > (size_t)SPLA_STATIC_WORKSPACE_BYTES) return SPLA_ERR_CAPACITY;
    int dev = -1;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        spla::set_last_cuda_error((int32_t)e);
        return SPLA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return SPLA_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if ((st = static_ws_for(dev, &ws)) != SPLA_OK) return st;
    return spla_decode(params, cache, q, rms_gamma, out, sel_idx, o_sparse_dbg, o_rla_dbg, ws,
                       (size_t)SPLA_STATIC_WORKSPACE_BYTES, dev_status, stream);
}
