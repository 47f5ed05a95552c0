// Pieces shared by the two decode kernels (CUDA-core and tensor-core consumers):
// vector loads, the per-partition epilogue that merges the consumer warps'
// softmax states, and the log-sum-exp merge kernel across partitions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

template <typename T>
__device__ __forceinline__ void load16_f32(const T* p, float* f);

template <>
__device__ __forceinline__ void load16_f32<float>(const float* p, float* f)
{
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x;
    f[1] = v.y;
    f[2] = v.z;
    f[3] = v.w;
}

template <>
__device__ __forceinline__ void load16_f32<__nv_bfloat16>(const __nv_bfloat16* p, float* f)
{
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    bf16x2_to_f32(v.x, f[0], f[1]);
    bf16x2_to_f32(v.y, f[2], f[3]);
    bf16x2_to_f32(v.z, f[4], f[5]);
    bf16x2_to_f32(v.w, f[6], f[7]);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x)
{
    return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x)
{
    return __float2bfloat16_rn(x);
}

constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int cmax(int a, int b) { return a > b ? a : b; }

// Merges the NCW consumer warps' states (m: running max, l: softmax sum, acc:
// unnormalised output, all relative to m) of one (sequence, kv head, partition)
// and writes either the final output row (the sequence fits in one partition) or
// the partition's state to the workspace.
template <typename T, int D, int G, int NCW, int THREADS>
__device__ __forceinline__ void finish_partition(const DecodeArgs& a, const float* mg_m, const float* mg_l,
                                                 const float* mg_acc, int s, int kvh, int part, bool split)
{
    const int NP = a.num_partitions;
    for (int idx = threadIdx.x; idx < G * D; idx += THREADS) {
        const int g = idx / D;
        const int d = idx % D;
        float M = (-INFINITY);
#pragma unroll
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, mg_m[w * G + g]);
        float num = 0.f, den = 0.f;
        if (M != (-INFINITY)) {
#pragma unroll
            for (int w = 0; w < NCW; ++w) {
                const float mw = mg_m[w * G + g];
                if (mw != (-INFINITY)) {
                    const float sc = exp2f(mw - M);
                    num = fmaf(sc, mg_acc[(w * G + g) * D + d], num);
                    den = fmaf(sc, mg_l[w * G + g], den);
                }
            }
        }
        const int h = kvh * G + g;
        if (!split) {
            T* o = static_cast<T*>(a.out) + ((size_t)s * a.num_heads + h) * D;
            o[d] = from_f32<T>(den > 0.f ? num / den : 0.f);
        } else {
            const size_t row = ((size_t)s * a.num_heads + h) * NP + part;
            a.ws_acc[row * D + d] = num;
            if (d == 0) {
                a.ws_ml[row * 2] = M;
                a.ws_ml[row * 2 + 1] = den;
            }
        }
    }
}

// Log-sum-exp merge of the partitions of one (sequence, query head):
// M = max_p m_p, out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p.
template <typename T, int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeArgs a, int partition_tokens, int block_size)
{
    pdl_wait_primary();
    __shared__ float s_w[kMaxPartitions];
    __shared__ float s_red[4];
    __shared__ float s_den;
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    int L = __ldg(a.context_lens + s);
    const int Lcap = min(a.max_context_len, a.max_blocks_per_seq * block_size);
    L = L < 0 ? 0 : (L > Lcap ? Lcap : L);
    const int np = (L + partition_tokens - 1) / partition_tokens;
    if (np <= 1) return;  // written directly by the partition kernel
    const int NP = a.num_partitions;
    const size_t row0 = ((size_t)s * a.num_heads + h) * NP;
    const float* ml = a.ws_ml + row0 * 2;

    float M = -INFINITY;
    for (int p = threadIdx.x; p < np; p += blockDim.x) M = fmaxf(M, ml[2 * p]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = M;
    __syncthreads();
    M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
    __syncthreads();

    float den = 0.f;
    for (int p = threadIdx.x; p < np; p += blockDim.x) {
        const float mp = ml[2 * p];
        const float w = (mp == -INFINITY) ? 0.f : exp2f(mp - M);
        s_w[p] = w;
        den = fmaf(w, ml[2 * p + 1], den);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = den;
    __syncthreads();
    if (threadIdx.x == 0) s_den = s_red[0] + s_red[1] + s_red[2] + s_red[3];
    __syncthreads();
    const float inv = s_den > 0.f ? 1.f / s_den : 0.f;

    T* o = static_cast<T*>(a.out) + ((size_t)s * a.num_heads + h) * D;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float num = 0.f;
        const float* accp = a.ws_acc + row0 * D + d;
        for (int p = 0; p < np; ++p) num = fmaf(s_w[p], accp[(size_t)p * D], num);
        o[d] = from_f32<T>(num * inv);
    }
}

// Launches the merge kernel after a partition kernel with programmatic dependent
// launch: its CTAs may be scheduled while the partition kernel drains and wait
// (griddepcontrol.wait) until that kernel's writes are visible.
template <typename T, int D>
cudaError_t launch_merge(const DecodeArgs& a, int block_size, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_heads, a.num_seqs, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_merge_kernel<T, D>, a, a.partition_blocks * block_size, block_size);
}

}  // namespace
}  // namespace pa
