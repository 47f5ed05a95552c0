// C ABI of libpa.so (declared in include/pa.h): argument validation, dispatch to
// the kernels, the device status word, and the per-thread error message.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "pa.h"
#include "pa_internal.h"

namespace pa {

static thread_local std::string g_err;

void set_error(const std::string& msg) { g_err = msg; }

namespace {

// Device status word: kernels OR PA_DEV_* bits into it.  Host code reaches it
// through its per-device address (the symbol itself is only a host-side handle).
__device__ unsigned int g_status_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_status_ptr[kMaxDevices] = {};
unsigned long long g_status_ctx[kMaxDevices] = {};  // context id each cached address belongs to

pa_status cuda_fail(const char* what, cudaError_t e)
{
    set_error(std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
    return PA_ERR_CUDA;
}

// Address of the status word on the current device: resolved once per device and
// context, and again after a device reset has re-created the context.
pa_status status_ptr(unsigned int** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("device index out of range");
        return PA_ERR_INVALID;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_status_ptr[dev] || ctx == 0 || g_status_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_status_word);
        if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress(status word)", e);
        g_status_ptr[dev] = static_cast<unsigned int*>(p);
        g_status_ctx[dev] = current_context_id();  // current now, if it was not before the lookup
    }
    *out = g_status_ptr[dev];
    return PA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elt_bytes(pa_dtype dt) { return dt == PA_DTYPE_F32 ? 4 : 2; }

pa_status check_common(const char* fn, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                       pa_dtype dtype)
{
    if (dtype != PA_DTYPE_F32 && dtype != PA_DTYPE_BF16) {
        set_error(std::string(fn) + ": dtype must be PA_DTYPE_F32 or PA_DTYPE_BF16");
        return PA_ERR_UNSUPPORTED;
    }
    if (head_dim != 64 && head_dim != 128) {
        set_error(std::string(fn) + ": head_dim must be 64 or 128");
        return PA_ERR_UNSUPPORTED;
    }
    if (block_size != 16 && block_size != 32) {
        set_error(std::string(fn) + ": block_size must be 16 or 32");
        return PA_ERR_UNSUPPORTED;
    }
    if (num_kv_heads <= 0 || num_kv_heads > 65535 || num_blocks <= 0) {
        set_error(std::string(fn) + ": num_kv_heads and num_blocks must be > 0 (num_kv_heads <= 65535)");
        return PA_ERR_INVALID;
    }
    return PA_OK;
}

constexpr int kAutoPartitionTokens = 512;

// Partition tokens for the arguments, or a negative pa_status.
int resolve_partition(int block_size, int max_context_len, int partition_size)
{
    int p = partition_size > 0 ? partition_size : kAutoPartitionTokens;
    if (p % block_size != 0 || p > kMaxPartitionTokens) {
        set_error("partition_size must be a multiple of block_size and at most " +
                  std::to_string(kMaxPartitionTokens));
        return PA_ERR_INVALID;
    }
    const long np = ((long)max_context_len + p - 1) / p;
    if (np > kMaxPartitions) {
        set_error("max_context_len / partition_size exceeds " + std::to_string(kMaxPartitions) +
                  " partitions; use a larger partition_size");
        return PA_ERR_UNSUPPORTED;
    }
    return p;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_last_error_string(void) { return g_err.c_str(); }

int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                             int max_context_len, int partition_size)
{
    (void)num_seqs;
    (void)num_heads;
    (void)num_kv_heads;
    (void)head_dim;
    if (block_size != 16 && block_size != 32) {
        set_error("pa_decode_partition_size: block_size must be 16 or 32");
        return PA_ERR_UNSUPPORTED;
    }
    if (max_context_len < 0 || partition_size < 0) {
        set_error("pa_decode_partition_size: negative size");
        return PA_ERR_INVALID;
    }
    return resolve_partition(block_size, max_context_len, partition_size);
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                int max_context_len, int partition_size)
{
    const int p = pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                           max_context_len, partition_size);
    if (p <= 0 || num_seqs <= 0 || num_heads <= 0 || head_dim <= 0) return 0;
    const size_t np = max_context_len > 0 ? ((size_t)max_context_len + p - 1) / p : 1;
    return decode_workspace((size_t)num_seqs, (size_t)num_heads, (size_t)head_dim, np).total;
}

}  // extern "C"

namespace pa {
namespace {

// pa_decode, pa_decode_plan and pa_decode_run: the same checks and arguments, then the
// plan kernel, the persistent kernel and merge, or both.  The plan phase does not
// touch out, q or the caches (they may be null).
pa_status decode_call(const char* fn, int phases, void* out, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                      int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                      int num_blocks, int max_context_len, float scale, int partition_size, void* workspace,
                      size_t workspace_bytes, pa_dtype dtype, void* stream)
{
    const std::string name(fn);
    pa_status st = check_common(fn, num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (st != PA_OK) return st;
    if (num_seqs < 0 || num_seqs > 65535 || num_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 ||
        partition_size < 0 || !std::isfinite(scale)) {
        set_error(name + ": bad size or scale");
        return PA_ERR_INVALID;
    }
    if (num_heads % num_kv_heads != 0) {
        set_error(name + ": num_heads must be a multiple of num_kv_heads");
        return PA_ERR_INVALID;
    }
    const int group = num_heads / num_kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8) {
        set_error(name + ": num_heads / num_kv_heads must be 1, 2, 4 or 8");
        return PA_ERR_UNSUPPORTED;
    }
    if (num_seqs == 0) return PA_OK;
    const bool run = (phases & kDecodeRun) != 0;
    if ((run && (!out || !q || !k_cache || !v_cache)) || !block_tables || !context_lens) {
        set_error(name + ": null pointer");
        return PA_ERR_INVALID;
    }
    if ((run && (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4)) {
        set_error(name + ": misaligned pointer (q, out, caches need 16 bytes)");
        return PA_ERR_INVALID;
    }
    if (decode_uses_tensor_cores(dtype, head_dim, group) &&
        (int64_t)num_blocks * num_kv_heads * block_size > (int64_t)INT32_MAX) {
        set_error(name + ": num_blocks * num_kv_heads * block_size must stay below 2^31 (tensor-copy row index)");
        return PA_ERR_UNSUPPORTED;
    }
    const int p = resolve_partition(block_size, max_context_len, partition_size);
    if (p < 0) return (pa_status)p;
    const int np = max_context_len > 0 ? (max_context_len + p - 1) / p : 1;
    const DecodeWorkspace wl = decode_workspace((size_t)num_seqs, (size_t)num_heads, (size_t)head_dim, (size_t)np);
    if (!workspace || workspace_bytes < wl.total || !aligned(workspace, 16)) {
        set_error(name + ": workspace missing, too small (need " + std::to_string(wl.total) +
                  " bytes) or not 16-byte aligned");
        return PA_ERR_INVALID;
    }
    DecodeArgs a{};
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    a.plan = reinterpret_cast<unsigned int*>(ws + wl.plan);
    a.plan_list = reinterpret_cast<uint2*>(ws + wl.list);
    a.split_list = reinterpret_cast<uint2*>(ws + wl.splits);
    if (np > 1) {
        a.ws_acc = reinterpret_cast<float*>(ws + wl.acc);
        a.ws_ml = reinterpret_cast<float*>(ws + wl.ml);
    }
    unsigned int* status = nullptr;
    st = status_ptr(&status);
    if (st != PA_OK) return st;
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.status = status;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.max_context_len = max_context_len;
    a.partition_blocks = p / block_size;
    a.adaptive = partition_size == 0 ? 1 : 0;
    a.num_partitions = np;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.phases = phases;
    const cudaError_t e =
        launch_decode(a, dtype, head_dim, block_size, group, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail((name + " launch").c_str(), e);
    return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" {

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_heads,
                    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                    int max_context_len, float scale, int partition_size, void* workspace,
                    size_t workspace_bytes, pa_dtype dtype, void* stream)
{
    pa::CallRange range("pa_decode");
    return decode_call("pa_decode", kDecodePlan | kDecodeRun, out, q, k_cache, v_cache, block_tables, context_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       max_context_len, scale, partition_size, workspace, workspace_bytes, dtype, stream);
}

pa_status pa_decode_plan(const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                         int max_context_len, int partition_size, void* workspace, size_t workspace_bytes,
                         pa_dtype dtype, void* stream)
{
    pa::CallRange range("pa_decode_plan");
    return decode_call("pa_decode_plan", kDecodePlan, nullptr, nullptr, nullptr, nullptr, block_tables, context_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       max_context_len, 1.0f, partition_size, workspace, workspace_bytes, dtype, stream);
}

pa_status pa_decode_run(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_heads,
                        int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                        int max_context_len, float scale, int partition_size, void* workspace,
                        size_t workspace_bytes, pa_dtype dtype, void* stream)
{
    pa::CallRange range("pa_decode_run");
    return decode_call("pa_decode_run", kDecodeRun, out, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       max_context_len, scale, partition_size, workspace, workspace_bytes, dtype, stream);
}

pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                               int block_size, int num_blocks, pa_dtype dtype, void* stream)
{
    pa::CallRange range("pa_reshape_and_cache");
    pa_status st = check_common("pa_reshape_and_cache", num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (st != PA_OK) return st;
    if (num_tokens < 0) {
        set_error("pa_reshape_and_cache: num_tokens < 0");
        return PA_ERR_INVALID;
    }
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) {
        set_error("pa_reshape_and_cache: null pointer");
        return PA_ERR_INVALID;
    }
    if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8)) {
        set_error("pa_reshape_and_cache: misaligned pointer");
        return PA_ERR_INVALID;
    }
    unsigned int* status = nullptr;
    st = status_ptr(&status);
    if (st != PA_OK) return st;
    ReshapeArgs a{key, value, k_cache, v_cache, slot_mapping, status, num_tokens, num_kv_heads, num_blocks};
    const cudaError_t e =
        launch_reshape_and_cache(a, elt_bytes(dtype), head_dim, block_size, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("pa_reshape_and_cache launch", e);
    return PA_OK;
}

pa_status pa_check_block_mapping(const int64_t* block_mapping, int num_pairs, int num_blocks)
{
    if (num_pairs < 0 || num_blocks <= 0 || (num_pairs > 0 && !block_mapping)) {
        set_error("pa_check_block_mapping: bad count or null array");
        return PA_ERR_INVALID;
    }
    // (block, pair index) of every destination, then of every source, sorted by block
    std::vector<std::pair<int64_t, int>> dst, src;
    dst.reserve(num_pairs);
    src.reserve(num_pairs);
    for (int i = 0; i < num_pairs; ++i) {
        const int64_t s = block_mapping[2 * i], d = block_mapping[2 * i + 1];
        if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
            set_error("pa_check_block_mapping: pair " + std::to_string(i) + " names a block outside [0, num_blocks)");
            return PA_ERR_INVALID;
        }
        dst.emplace_back(d, i);
        src.emplace_back(s, i);
    }
    std::sort(dst.begin(), dst.end());
    std::sort(src.begin(), src.end());
    for (size_t k = 1; k < dst.size(); ++k)
        if (dst[k].first == dst[k - 1].first) {
            set_error("pa_check_block_mapping: pairs " + std::to_string(dst[k - 1].second) + " and " +
                      std::to_string(dst[k].second) + " write the same block " + std::to_string(dst[k].first));
            return PA_ERR_INVALID;
        }
    for (size_t k = 0, m = 0; k < dst.size(); ++k) {
        while (m < src.size() && src[m].first < dst[k].first) ++m;
        if (m < src.size() && src[m].first == dst[k].first) {
            set_error("pa_check_block_mapping: block " + std::to_string(dst[k].first) + " is written by pair " +
                      std::to_string(dst[k].second) + " and read by pair " + std::to_string(src[m].second));
            return PA_ERR_INVALID;
        }
    }
    return PA_OK;
}

pa_status pa_check_slot_mapping(const int64_t* slot_mapping, int num_tokens, int num_blocks, int block_size)
{
    if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || (num_tokens > 0 && !slot_mapping)) {
        set_error("pa_check_slot_mapping: bad count or size, or null array");
        return PA_ERR_INVALID;
    }
    const int64_t nslots = (int64_t)num_blocks * block_size;
    std::vector<std::pair<int64_t, int>> slots;
    slots.reserve(num_tokens);
    for (int t = 0; t < num_tokens; ++t) {
        const int64_t s = slot_mapping[t];
        if (s < 0) continue;  // padding
        if (s >= nslots) {
            set_error("pa_check_slot_mapping: token " + std::to_string(t) + " has slot " + std::to_string(s) +
                      ", past the pool's " + std::to_string(nslots) + " slots");
            return PA_ERR_INVALID;
        }
        slots.emplace_back(s, t);
    }
    std::sort(slots.begin(), slots.end());
    for (size_t k = 1; k < slots.size(); ++k)
        if (slots[k].first == slots[k - 1].first) {
            set_error("pa_check_slot_mapping: tokens " + std::to_string(slots[k - 1].second) + " and " +
                      std::to_string(slots[k].second) + " share slot " + std::to_string(slots[k].first));
            return PA_ERR_INVALID;
        }
    return PA_OK;
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping, int num_pairs,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                         void* stream)
{
    pa::CallRange range("pa_copy_blocks");
    pa_status st = check_common("pa_copy_blocks", num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (st != PA_OK) return st;
    if (num_pairs < 0 || num_pairs > 65535) {
        set_error("pa_copy_blocks: num_pairs must be in [0, 65535]");
        return PA_ERR_INVALID;
    }
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !block_mapping) {
        set_error("pa_copy_blocks: null pointer");
        return PA_ERR_INVALID;
    }
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_mapping, 8)) {
        set_error("pa_copy_blocks: misaligned pointer");
        return PA_ERR_INVALID;
    }
    unsigned int* status = nullptr;
    st = status_ptr(&status);
    if (st != PA_OK) return st;
    CopyArgs a{};
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_mapping = block_mapping;
    a.status = status;
    a.num_pairs = num_pairs;
    a.num_blocks = num_blocks;
    a.block_bytes = (size_t)num_kv_heads * block_size * head_dim * elt_bytes(dtype);
    const cudaError_t e = launch_copy_blocks(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("pa_copy_blocks launch", e);
    return PA_OK;
}

static pa_status prefill_impl(const char* name, void* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables,
                     const int32_t* context_lens, const int32_t* q_start, int num_seqs, int num_heads,
                     int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                     int num_query_tokens, int max_query_len, float scale, pa_dtype dtype, void* stream,
                              void* workspace, size_t workspace_bytes)
{
    pa::CallRange range(name);
    pa_status st = check_common("pa_prefill", num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (st != PA_OK) return st;
    if (dtype != PA_DTYPE_BF16 || head_dim != 128) {
        set_error("pa_prefill: bf16 with head_dim 128 only (the tensor-core tile)");
        return PA_ERR_UNSUPPORTED;
    }
    if (num_seqs < 0 || num_seqs > 65535 || num_heads <= 0 || num_heads % num_kv_heads != 0 ||
        num_query_tokens < 0 || max_query_len < 0 || max_blocks_per_seq < 0 || !(scale == scale) ||
        scale == INFINITY || scale == -INFINITY) {
        set_error("pa_prefill: bad sizes or scale");
        return PA_ERR_INVALID;
    }
    const int group = num_heads / num_kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8) {
        set_error("pa_prefill: num_heads / num_kv_heads must be 1, 2, 4 or 8");
        return PA_ERR_UNSUPPORTED;
    }
    if (workspace && (workspace_bytes < pa_prefill_workspace_size() || !aligned(workspace, 16))) {
        set_error("pa_prefill_ws: workspace smaller than pa_prefill_workspace_size() or not 16-byte aligned");
        return PA_ERR_INVALID;
    }
    if (num_seqs == 0 || num_query_tokens == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !q_start) {
        set_error("pa_prefill: null pointer");
        return PA_ERR_INVALID;
    }
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16)) {
        set_error("pa_prefill: misaligned pointer (q, out, caches need 16 bytes)");
        return PA_ERR_INVALID;
    }
    if ((int64_t)num_blocks * num_kv_heads * block_size > (int64_t)INT32_MAX) {
        set_error("pa_prefill: num_blocks * num_kv_heads * block_size must stay below 2^31 (tensor-copy row index)");
        return PA_ERR_UNSUPPORTED;
    }
    unsigned int* status = nullptr;
    st = status_ptr(&status);
    if (st != PA_OK) return st;
    PrefillArgs a{};
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.q_start = q_start;
    a.status = status;
    a.sched = static_cast<unsigned int*>(workspace);
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.num_query_tokens = num_query_tokens;
    a.max_query_len = max_query_len;
    a.scale_log2 = scale * 1.4426950408889634f;
    if (workspace) {
        // the item counter starts at zero on every call, in stream order
        const cudaError_t z = cudaMemsetAsync(workspace, 0, sizeof(unsigned int), static_cast<cudaStream_t>(stream));
        if (z != cudaSuccess) return cuda_fail("pa_prefill_ws counter reset", z);
    }
    const cudaError_t e =
        launch_prefill(a, group, num_query_tokens, max_query_len, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("pa_prefill launch", e);
    return PA_OK;
}

size_t pa_prefill_workspace_size(void) { return 256; }

pa_status pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, const int32_t* q_start, int num_seqs, int num_heads,
                     int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                     int num_query_tokens, int max_query_len, float scale, pa_dtype dtype, void* stream)
{
    return prefill_impl("pa_prefill", out, q, k_cache, v_cache, block_tables, context_lens, q_start, num_seqs,
                        num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                        num_query_tokens, max_query_len, scale, dtype, stream, nullptr, 0);
}

pa_status pa_prefill_ws(void* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, const int32_t* context_lens, const int32_t* q_start,
                        int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                        int max_blocks_per_seq, int num_blocks, int num_query_tokens, int max_query_len, float scale,
                        void* workspace, size_t workspace_bytes, pa_dtype dtype, void* stream)
{
    if (!workspace) {
        set_error("pa_prefill_ws: null workspace");
        return PA_ERR_INVALID;
    }
    return prefill_impl("pa_prefill_ws", out, q, k_cache, v_cache, block_tables, context_lens, q_start, num_seqs,
                        num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                        num_query_tokens, max_query_len, scale, dtype, stream, workspace, workspace_bytes);
}

// Address a kernel can use for p: device memory as is, pinned (page-locked) host
// memory through its device mapping; anything else is refused.
static pa_status kernel_address(const char* who, const char* what, const void* p, const void** out)
{
    cudaPointerAttributes at{};
    const cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        set_error(std::string(who) + ": cannot query " + what + ": " + cudaGetErrorString(e));
        return PA_ERR_INVALID;
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
        *out = p;
        return PA_OK;
    }
    if (at.type == cudaMemoryTypeHost && at.devicePointer) {
        *out = at.devicePointer;
        return PA_OK;
    }
    set_error(std::string(who) + ": " + what + " must be device memory or pinned host memory");
    return PA_ERR_INVALID;
}

pa_status pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, const void* src_k_cache, const void* src_v_cache,
                         const int64_t* block_mapping, int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_src_blocks, int num_dst_blocks, pa_dtype dtype, void* stream)
{
    pa::CallRange range("pa_swap_blocks");
    pa_status st = check_common("pa_swap_blocks", num_kv_heads, head_dim, block_size, num_src_blocks, dtype);
    if (st != PA_OK) return st;
    if (num_dst_blocks <= 0) {
        set_error("pa_swap_blocks: num_dst_blocks must be > 0");
        return PA_ERR_INVALID;
    }
    if (num_pairs < 0 || num_pairs > 65535) {
        set_error("pa_swap_blocks: num_pairs must be in [0, 65535]");
        return PA_ERR_INVALID;
    }
    if (num_pairs == 0) return PA_OK;
    if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !block_mapping) {
        set_error("pa_swap_blocks: null pointer");
        return PA_ERR_INVALID;
    }
    if (!aligned(dst_k_cache, 16) || !aligned(dst_v_cache, 16) || !aligned(src_k_cache, 16) ||
        !aligned(src_v_cache, 16) || !aligned(block_mapping, 8)) {
        set_error("pa_swap_blocks: misaligned pointer");
        return PA_ERR_INVALID;
    }
    SwapArgs a{};
    const void* p = nullptr;
    if ((st = kernel_address("pa_swap_blocks", "dst_k_cache", dst_k_cache, &p)) != PA_OK) return st;
    a.dst_k = const_cast<void*>(p);
    if ((st = kernel_address("pa_swap_blocks", "dst_v_cache", dst_v_cache, &p)) != PA_OK) return st;
    a.dst_v = const_cast<void*>(p);
    if ((st = kernel_address("pa_swap_blocks", "src_k_cache", src_k_cache, &a.src_k)) != PA_OK) return st;
    if ((st = kernel_address("pa_swap_blocks", "src_v_cache", src_v_cache, &a.src_v)) != PA_OK) return st;
    if ((st = kernel_address("pa_swap_blocks", "block_mapping", block_mapping, &p)) != PA_OK) return st;
    a.block_mapping = static_cast<const int64_t*>(p);
    unsigned int* status = nullptr;
    st = status_ptr(&status);
    if (st != PA_OK) return st;
    a.status = status;
    a.num_pairs = num_pairs;
    a.num_src_blocks = num_src_blocks;
    a.num_dst_blocks = num_dst_blocks;
    a.block_bytes = (size_t)num_kv_heads * block_size * head_dim * elt_bytes(dtype);
    const cudaError_t e = launch_swap_blocks(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("pa_swap_blocks launch", e);
    return PA_OK;
}

pa_status pa_selftest_bounded_wait(uint64_t* waited_ns, void* stream)
{
    unsigned int* status = nullptr;
    pa_status st = status_ptr(&status);
    if (st != PA_OK) return st;
    unsigned long long ns = 0;
    const cudaError_t e = launch_wait_selftest(status, &ns, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("pa_selftest_bounded_wait", e);
    if (waited_ns) *waited_ns = (uint64_t)ns;
    return PA_OK;
}

pa_status pa_device_status(uint32_t* flags, void* stream)
{
    if (!flags) return PA_ERR_INVALID;
    unsigned int* status = nullptr;
    pa_status st = status_ptr(&status);
    if (st != PA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, status, sizeof(v), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail("pa_device_status read", e);
    e = cudaMemsetAsync(status, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return cuda_fail("pa_device_status clear", e);
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail("pa_device_status sync", e);
    *flags = v;
    return PA_OK;
}

}  // extern "C"
