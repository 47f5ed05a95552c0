// The two companions of the decode kernel, for sm_100a.
//
// reshape_and_cache: the slot-mapped KV append.  The new token's K and V rows are
// written to slot T[b]*B + o of the pools ("PagedAttention Paper Breakdown",
// section 2, Address Translation Formula); the caller passes that slot per token.
// copy_blocks: the copy-on-write block copy ("PagedAttention and vLLM
// Architecture", section 3): a shared block about to be written is duplicated
// into a fresh block before the write.
// swap_blocks: whole blocks between a device pool and a pinned host pool
// ("PagedAttention Paper Breakdown", "Engineering Limitations": CPU-GPU block
// swapping under memory pressure).
//
// Both are pure data movement, bounded by HBM bandwidth: every thread moves
// 16-byte vectors, consecutive threads cover consecutive bytes of a row (or of a
// block), and indices are range-checked on the device (bad ones raise a status bit
// and are skipped, never dereferenced).
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_internal.h"

namespace pa {

namespace {

// One thread per 16-byte chunk of one (token, kv head) row, for K and for V.
template <int CPR>  // 16-byte chunks per row
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const ReshapeArgs a, int block_size)
{
    const int64_t total = (int64_t)a.num_tokens * a.num_kv_heads * CPR;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += stride) {
        const int chunk = (int)(idx % CPR);
        const int64_t th = idx / CPR;                 // token * kv_heads + head
        const int h = (int)(th % a.num_kv_heads);
        const int64_t t = th / a.num_kv_heads;
        const int64_t slot = __ldg(a.slot_mapping + t);
        if (slot < 0) continue;                        // padding token
        if (slot >= (int64_t)a.num_blocks * block_size) {
            if (chunk == 0 && h == 0) atomicOr(a.status, PA_DEV_BAD_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot % block_size;
        const int64_t dst = ((blk * a.num_kv_heads + h) * block_size + off) * CPR + chunk;
        const int64_t src = th * CPR + chunk;
        const uint4 kv = __ldg(reinterpret_cast<const uint4*>(a.key) + src);
        const uint4 vv = __ldg(reinterpret_cast<const uint4*>(a.value) + src);
        reinterpret_cast<uint4*>(a.k_cache)[dst] = kv;
        reinterpret_cast<uint4*>(a.v_cache)[dst] = vv;
    }
}

// grid: (chunks of a block, pair, 2 pools).  Each thread copies kVec 16-byte vectors.
constexpr int kCopyThreads = 256;
constexpr int kCopyVec = 4;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const CopyArgs a)
{
    const int pair = blockIdx.y;
    const int64_t src = __ldg(a.block_mapping + 2 * pair);
    const int64_t dst = __ldg(a.block_mapping + 2 * pair + 1);
    if (src < 0 || dst < 0 || src >= a.num_blocks || dst >= a.num_blocks) {
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) atomicOr(a.status, PA_DEV_BAD_PAIR);
        return;
    }
    char* pool = static_cast<char*>(blockIdx.z == 0 ? a.k_cache : a.v_cache);
    const uint4* s = reinterpret_cast<const uint4*>(pool + (size_t)src * a.block_bytes);
    uint4* d = reinterpret_cast<uint4*>(pool + (size_t)dst * a.block_bytes);
    const int64_t nvec = (int64_t)(a.block_bytes / 16);
    const int64_t base = (int64_t)blockIdx.x * kCopyThreads * kCopyVec + threadIdx.x;
    uint4 buf[kCopyVec];
#pragma unroll
    for (int k = 0; k < kCopyVec; ++k) {
        const int64_t i = base + (int64_t)k * kCopyThreads;
        if (i < nvec) buf[k] = s[i];
    }
#pragma unroll
    for (int k = 0; k < kCopyVec; ++k) {
        const int64_t i = base + (int64_t)k * kCopyThreads;
        if (i < nvec) d[i] = buf[k];
    }
}

// Block swap between a device pool and a pinned host pool (either direction), the
// host side reached through its device mapping over PCIe.  Same tiling as the
// copy-on-write copy; plain loads and stores (the host side is not read-only cached).
__global__ void __launch_bounds__(kCopyThreads) swap_blocks_kernel(const SwapArgs a)
{
    const int pair = blockIdx.y;
    const int64_t src = a.block_mapping[2 * pair];
    const int64_t dst = a.block_mapping[2 * pair + 1];
    if (src < 0 || dst < 0 || src >= a.num_src_blocks || dst >= a.num_dst_blocks) {
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) atomicOr(a.status, PA_DEV_BAD_PAIR);
        return;
    }
    const char* sp = static_cast<const char*>(blockIdx.z == 0 ? a.src_k : a.src_v);
    char* dp = static_cast<char*>(blockIdx.z == 0 ? a.dst_k : a.dst_v);
    const uint4* s = reinterpret_cast<const uint4*>(sp + (size_t)src * a.block_bytes);
    uint4* d = reinterpret_cast<uint4*>(dp + (size_t)dst * a.block_bytes);
    const int64_t nvec = (int64_t)(a.block_bytes / 16);
    const int64_t base = (int64_t)blockIdx.x * kCopyThreads * kCopyVec + threadIdx.x;
    uint4 buf[kCopyVec];
#pragma unroll
    for (int k = 0; k < kCopyVec; ++k) {
        const int64_t i = base + (int64_t)k * kCopyThreads;
        if (i < nvec) buf[k] = s[i];
    }
#pragma unroll
    for (int k = 0; k < kCopyVec; ++k) {
        const int64_t i = base + (int64_t)k * kCopyThreads;
        if (i < nvec) d[i] = buf[k];
    }
}

}  // namespace

cudaError_t launch_reshape_and_cache(const ReshapeArgs& a, int elt_bytes, int head_dim, int block_size,
                                     cudaStream_t stream)
{
    const int cpr = head_dim * elt_bytes / 16;
    const int64_t total = (int64_t)a.num_tokens * a.num_kv_heads * cpr;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 64) blocks = 148 * 64;  // grid-stride beyond ~64 CTAs per SM
    switch (cpr) {
        case 8: reshape_and_cache_kernel<8><<<(unsigned)blocks, threads, 0, stream>>>(a, block_size); break;
        case 16: reshape_and_cache_kernel<16><<<(unsigned)blocks, threads, 0, stream>>>(a, block_size); break;
        case 32: reshape_and_cache_kernel<32><<<(unsigned)blocks, threads, 0, stream>>>(a, block_size); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_copy_blocks(const CopyArgs& a, cudaStream_t stream)
{
    if (a.num_pairs == 0) return cudaSuccess;
    const int64_t nvec = (int64_t)(a.block_bytes / 16);
    const int64_t per_cta = (int64_t)kCopyThreads * kCopyVec;
    dim3 grid((unsigned)((nvec + per_cta - 1) / per_cta), (unsigned)a.num_pairs, 2);
    copy_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_swap_blocks(const SwapArgs& a, cudaStream_t stream)
{
    if (a.num_pairs == 0) return cudaSuccess;
    const int64_t nvec = (int64_t)(a.block_bytes / 16);
    const int64_t per_cta = (int64_t)kCopyThreads * kCopyVec;
    dim3 grid((unsigned)((nvec + per_cta - 1) / per_cta), (unsigned)a.num_pairs, 2);
    swap_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace pa
