// tri_static_scratch.cu - tri_compress_step for callers that cannot allocate.
//
// Some callers have no way to obtain device scratch memory: a serving engine
// that reserves nearly all of HBM for its paged KV block pool at start-up
// and forbids allocation on the decode path, or a plain-C plugin loaded into
// such an engine with no allocator handle of its own.  tri_compress_step
// needs a caller-provided workspace; this entry point instead uses one
// fixed array of device memory that is part of the library image itself.
//
// The array lives at file scope below.  Every GPU that loads this library
// holds it (TRI_STATIC_SCRATCH_BYTES) until the process exits.  Host code
// cannot use the array's name as a device address, so the address is looked
// up with cudaGetSymbolAddress, with the device current, and cached.
//
// The array belongs to the CUDA context the library's module is loaded in:
// if that context is destroyed (cudaDeviceReset, or a reset of the device's
// primary context by any other code in the process) a new context holds a
// new copy of the array, possibly at another address.  The cache is
// therefore keyed by the unique id of the current context (cuCtxGetId), not
// by the device ordinal: a call made in a context other than the one the
// cached address came from looks the address up again.
#include <mutex>

#include <cuda.h>

#include "tri_attention.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[TRI_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;

struct CachedAddress {
    unsigned long long ctx_id;   // unique id of the context the address belongs to (0: none)
    void* addr;
};

std::mutex g_mu;
CachedAddress g_cache[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Driver entry points that name the current context (looked up once).
bool context_entry_points(CtxGetCurrentFn& get_current, CtxGetIdFn& get_id) {
    static CtxGetCurrentFn s_current = nullptr;
    static CtxGetIdFn s_id = nullptr;
    static bool tried = false;
    if (!tried) {   // called with g_mu held
        tried = true;
        void* a = nullptr;
        void* b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            s_current = reinterpret_cast<CtxGetCurrentFn>(a);
            s_id = reinterpret_cast<CtxGetIdFn>(b);
        }
    }
    get_current = s_current;
    get_id = s_id;
    return s_current != nullptr && s_id != nullptr;
}

// Unique id of the calling thread's current context; false if there is none
// or it cannot be named (then nothing is cached).
bool current_context_id(unsigned long long& id) {
    CtxGetCurrentFn get_current;
    CtxGetIdFn get_id;
    if (!context_entry_points(get_current, get_id)) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, &id) == CUDA_SUCCESS && id != 0;
}

// Device address of g_scratch in the current context.
tri_status scratch_in_current_context(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TRI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    unsigned long long id = 0;
    if (current_context_id(id) && g_cache[dev].ctx_id == id && g_cache[dev].addr != nullptr) {
        *out = g_cache[dev].addr;
        return TRI_OK;
    }
    void* p = nullptr;
    // The lookup makes the device's context current if no context was yet.
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return TRI_ERR_CUDA;
    if (current_context_id(id)) {
        g_cache[dev].ctx_id = id;
        g_cache[dev].addr = p;
    } else {
        g_cache[dev].ctx_id = 0;    // cannot tell contexts apart: look up on every call
        g_cache[dev].addr = nullptr;
    }
    *out = p;
    return TRI_OK;
}

}  // namespace

extern "C" size_t tri_static_scratch_bytes(void) { return (size_t)TRI_STATIC_SCRATCH_BYTES; }

extern "C" tri_status tri_compress_step_static_scratch(tri_kv_desc* desc, const float* qbar, const float* qabs,
                                                       const float* R, double rope_base, const int32_t* deltas,
                                                       int n_deltas, int budget, int window, int32_t* freed_ids,
                                                       int32_t* freed_count, int32_t* idx_out,
                                                       cudaStream_t stream) {
    const size_t need = tri_workspace_size(desc, budget);
    if (need > (size_t)TRI_STATIC_SCRATCH_BYTES) return TRI_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (need > 0) {
        const tri_status st = scratch_in_current_context(&ws);
        if (st != TRI_OK) return st;
    }
    // need == 0 means the descriptor or the budget is invalid:
    // tri_compress_step reports why before touching the workspace.
    return tri_compress_step(desc, qbar, qabs, R, rope_base, deltas, n_deltas, budget, window, freed_ids,
                             freed_count, idx_out, ws, (size_t)TRI_STATIC_SCRATCH_BYTES, nullptr, stream);
}
