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
// up with cudaGetSymbolAddress once per device, with that device current,
// on the first call made there, and cached.
#include <mutex>

#include "tri_attention.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[TRI_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_scratch on the current device (first call per device
// performs the lookup).
tri_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TRI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return TRI_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return TRI_OK;
}

}  // namespace

extern "C" tri_status tri_compress_step_static_scratch(tri_kv_desc* desc, const float* qbar, const float* qabs,
                                                       const float* R, double rope_base, const int32_t* deltas,
                                                       int n_deltas, int budget, int window, int32_t* freed_ids,
                                                       int32_t* freed_count, int32_t* idx_out,
                                                       cudaStream_t stream) {
    const size_t need = tri_workspace_size(desc, budget);
    if (need > (size_t)TRI_STATIC_SCRATCH_BYTES) return TRI_ERR_UNSUPPORTED;
    void* ws = nullptr;
    if (need > 0) {
        const tri_status st = scratch_on_current_device(&ws);
        if (st != TRI_OK) return st;
    }
    // need == 0 means the descriptor is invalid: tri_compress_step reports why.
    return tri_compress_step(desc, qbar, qabs, R, rope_base, deltas, n_deltas, budget, window, freed_ids,
                             freed_count, idx_out, ws, (size_t)TRI_STATIC_SCRATCH_BYTES, nullptr, stream);
}
