// Internal launch interface between the C-ABI layer (pa_api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "pa.h"

namespace pa {

// A profiler range (NVTX, header-only v3) around one C-ABI call, so a profiler can
// pick out pa_decode, pa_prefill and the companions by name.  With no profiler
// attached the push and pop are calls into the NVTX no-op stubs.
struct CallRange {
    explicit CallRange(const char* name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange&) = delete;
    CallRange& operator=(const CallRange&) = delete;
};

// Largest context partition (tokens) and largest number of partitions per sequence.
constexpr int kMaxPartitionTokens = 4096;
constexpr int kMaxPartitions = 2048;

struct DecodeArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    unsigned int* plan;        // [0] work counter, [1] (sequence, partition) pairs, [2] blocks per
                               // partition, [3] sequences split into several partitions, [4] CTAs
                               // that stopped taking units in the current run
    uint2* plan_list;          // [S * NP] longest first: {sequence << 11 | partition, context length}
    uint2* split_list;         // [S] the sequences split into several partitions (plan[3] of them):
                               // {sequence, context length}
    float* ws_acc;             // [S][Hq][NP][D] unnormalised partition outputs (NP > 1)
    float* ws_ml;              // [S][Hq][NP][2] (running max in log2 units, softmax sum)
    unsigned int* status;      // device status word (PA_DEV_* bits)
    int num_seqs;
    int num_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int num_blocks;
    int max_context_len;
    int partition_blocks;      // blocks per context partition (the smallest the plan may use)
    int adaptive;              // non-zero: the plan may use a multiple of partition_blocks
    int num_ctas;              // CTAs of the persistent kernel
    int first_wave;            // units the CTAs start on without waiting for the plan: CTA b < first_wave
                               // takes kv head b % Hkv of partition 0 of sequence b / Hkv (0: none)
    int num_partitions;        // NP = ceil(max_context_len / smallest partition tokens)
    float scale_log2;          // scale * log2(e): logits are kept in base-2 units
    int phases;                // host side: kDecodePlan and/or kDecodeRun
};

constexpr int kDecodePlan = 1;  // the plan kernel: work list into the workspace
constexpr int kDecodeRun = 2;   // the persistent kernel and the merge, from that work list

// Byte layout of the decode workspace: the work plan, then (when a sequence may
// span several partitions) the partition states.
struct DecodeWorkspace {
    size_t plan;       // 32 bytes: counter, pair count, blocks per partition, split count, exit count
    size_t list;       // 8 * S * NP bytes
    size_t splits;     // 8 * S bytes
    size_t acc;        // 4 * S * Hq * NP * D bytes (0 bytes when NP == 1)
    size_t ml;         // 8 * S * Hq * NP bytes (0 bytes when NP == 1)
    size_t total;
};

inline DecodeWorkspace decode_workspace(size_t S, size_t Hq, size_t D, size_t NP)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const bool split = NP > 1;
    DecodeWorkspace w{};
    w.plan = 0;
    w.list = 32;
    w.splits = up(w.list + 8 * S * NP);
    w.acc = up(w.splits + 8 * S);
    w.ml = up(w.acc + (split ? 4 * S * Hq * NP * D : 0));
    w.total = up(w.ml + (split ? 8 * S * Hq * NP : 0));
    return w;
}

// One call: the plan kernel, the persistent kernel (tensor cores for bf16 with a group
// of 2, 4 or 8 query heads per kv head, CUDA cores otherwise) and, when a sequence may
// span several partitions, the log-sum-exp merge kernel.
cudaError_t launch_decode(const DecodeArgs& a, pa_dtype dtype, int head_dim, int block_size, int group,
                          cudaStream_t stream);
bool decode_uses_tensor_cores(pa_dtype dtype, int head_dim, int group);

// Tensor maps (TMA descriptors).  The driver's encoder, looked up once, and a cached
// 2-D bf16 map of a pool [num_blocks][kv_heads][B][D] seen as `rows` rows of D
// elements, boxes of 64 columns x `box_rows` rows, 128-byte swizzle.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
cudaError_t tensor_map(CUtensorMap* out, const void* pool, uint64_t rows, int D, int box_rows);

// Process-unique id of the CUDA context current on this thread (cuCtxGetId), or 0
// when none is current or the driver lacks the call.  Device addresses of the
// library's own __device__ variables are cached per device under this id: a device
// reset re-creates the context (and may reload the module elsewhere), which changes
// the id, so the address is looked up again.
unsigned long long current_context_id();

struct ReshapeArgs {
    const void* key;
    const void* value;
    void* k_cache;
    void* v_cache;
    const int64_t* slot_mapping;
    unsigned int* status;
    int num_tokens;
    int num_kv_heads;
    int num_blocks;
};

cudaError_t launch_reshape_and_cache(const ReshapeArgs& a, int elt_bytes, int head_dim, int block_size,
                                     cudaStream_t stream);

struct CopyArgs {
    void* k_cache;
    void* v_cache;
    const int64_t* block_mapping;
    unsigned int* status;
    int num_pairs;
    int num_blocks;
    size_t block_bytes;        // num_kv_heads * block_size * head_dim * elt
};

cudaError_t launch_copy_blocks(const CopyArgs& a, cudaStream_t stream);

// Chunked prefill on the tensor cores (pa_prefill.cu): bf16, head_dim 128.
struct PrefillArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* q_start;    // [S + 1] query rows of each sequence
    unsigned int* status;
    unsigned int* sched;       // item counter (zero at launch) for a grid of one CTA per SM; null: one item per CTA
    int num_seqs;
    int num_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int num_blocks;
    int block_size;
    int num_query_tokens;      // rows of q and out: every sequence's rows must lie in [0, this)
    int max_query_len;         // the launch covers this many rows per sequence
    float scale_log2;
};

cudaError_t launch_prefill(const PrefillArgs& a, int group, int num_query_tokens, int max_query_len,
                           cudaStream_t stream);

// Whole-block copies between two pools, either of which may be pinned host memory
// (addressed through its device mapping).
struct SwapArgs {
    void* dst_k;
    void* dst_v;
    const void* src_k;
    const void* src_v;
    const int64_t* block_mapping;  // [num_pairs][2] (src block, dst block)
    unsigned int* status;
    int num_pairs;
    int num_src_blocks;
    int num_dst_blocks;
    size_t block_bytes;
};

cudaError_t launch_swap_blocks(const SwapArgs& a, cudaStream_t stream);

// One bounded wait on an mbarrier nothing arrives at (pa_selftest.cu); blocks until done.
cudaError_t launch_wait_selftest(unsigned int* status, unsigned long long* waited_ns, cudaStream_t stream);

}  // namespace pa
