// pa_decode_static_workspace: paged decode attention for callers that cannot
// allocate device memory.
//
// Some callers have no way to allocate: a plugin or script runtime that only hands
// out pointers to tensors it already owns, a process whose allocator is off limits
// (a frozen memory pool, a custom caching allocator that must not be bypassed), or
// code that must never call into the allocator on a latency-critical path.  This
// entry point takes the same inputs and output as pa_decode and uses, as its
// workspace, a fixed array in device memory that belongs to the library.
//
// The array is file-scope device memory: every GPU that loads the library holds
// PA_STATIC_WORKSPACE_BYTES of it until the process exits.  In host code the
// array's name is only a host-side handle, not a device address, so this file
// resolves the address once per device (cudaGetSymbolAddress, with that device
// current) on the first call made on the device, and passes that address on; a
// device reset makes the next call resolve it again.
// Nothing else here allocates.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "pa.h"
#include "pa_internal.h"

namespace pa {
void set_error(const std::string& msg);
}

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};
unsigned long long g_ws_ctx[kMaxDevices] = {};  // context id each cached address belongs to

// Device address of the array on the current device: resolved at the first call on
// the device, and again at the first call after a device reset (cudaDeviceReset
// ends the context; the next one may load the library's module at another address).
pa_status static_workspace(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        pa::set_error(std::string("pa_decode_static_workspace: cudaGetDevice: ") + cudaGetErrorString(e));
        return PA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        pa::set_error("pa_decode_static_workspace: device index out of range");
        return PA_ERR_INVALID;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    const unsigned long long ctx = pa::current_context_id();
    if (!g_ws_ptr[dev] || ctx == 0 || g_ws_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess || !p) {
            pa::set_error(std::string("pa_decode_static_workspace: cudaGetSymbolAddress: ") + cudaGetErrorString(e));
            return PA_ERR_CUDA;
        }
        g_ws_ptr[dev] = p;
        g_ws_ctx[dev] = pa::current_context_id();
    }
    *out = g_ws_ptr[dev];
    return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode_static_workspace(void* out, const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                                     int num_heads, int num_kv_heads, int head_dim, int block_size,
                                     int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                                     int partition_size, pa_dtype dtype, void* stream)
{
    pa::CallRange range("pa_decode_static_workspace");
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                 max_context_len, partition_size);
    if (need > (size_t)PA_STATIC_WORKSPACE_BYTES) {
        pa::set_error("pa_decode_static_workspace: these arguments need " + std::to_string(need) +
                      " bytes of workspace, more than the library's fixed " +
                      std::to_string((size_t)PA_STATIC_WORKSPACE_BYTES) +
                      " bytes; use pa_decode with a caller-owned workspace (or a larger partition_size)");
        return PA_ERR_UNSUPPORTED;
    }
    void* ws = nullptr;
    if (num_seqs > 0) {
        const pa_status st = static_workspace(&ws);
        if (st != PA_OK) return st;
    }
    return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads, num_kv_heads,
                     head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale, partition_size,
                     ws, (size_t)PA_STATIC_WORKSPACE_BYTES, dtype, stream);
}

}  // extern "C"
