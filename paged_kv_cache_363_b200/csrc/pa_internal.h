// Internal launch interface between the C-ABI layer (pa_api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "pa.h"

namespace pa {

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
    float* ws_acc;             // [S][Hq][NP][D] unnormalised partition outputs
    float* ws_ml;              // [S][Hq][NP][2] (running max in log2 units, softmax sum)
    unsigned int* status;      // device status word (PA_DEV_* bits)
    int num_seqs;
    int num_heads;
    int num_kv_heads;
    int max_blocks_per_seq;
    int num_blocks;
    int max_context_len;
    int partition_blocks;      // blocks per context partition
    int num_partitions;        // NP = ceil(max_context_len / partition tokens)
    float scale_log2;          // scale * log2(e): logits are kept in base-2 units
};

cudaError_t launch_decode(const DecodeArgs& a, pa_dtype dtype, int head_dim, int block_size, int group,
                          cudaStream_t stream);

// bf16 with a group of 2, 4 or 8 query heads per kv head runs on the tensor cores
// (pa_decode_mma.cu); everything else on the CUDA cores (pa_decode.cu).
bool decode_uses_tensor_cores(pa_dtype dtype, int head_dim, int group);
cudaError_t launch_decode_mma(const DecodeArgs& a, int head_dim, int block_size, int group, cudaStream_t stream);

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

}  // namespace pa
