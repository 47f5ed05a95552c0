// Pieces of the paged decode path shared by its two consumers (CUDA cores and
// tensor cores): vector loads, the longest-first work plan, the per-partition
// epilogue that merges the consumer warps' softmax states, and the log-sum-exp
// merge of a sequence's context partitions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

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

// Context length of sequence s as the kernels use it: clamped to what the launch
// covers (a value outside [0, Lcap] raises PA_DEV_BAD_CONTEXT where flag is set).
__device__ __forceinline__ int clamped_context(const DecodeArgs& a, int s, int block_size, bool flag)
{
    int L = __ldg(a.context_lens + s);
    const int Lcap = min(a.max_context_len, a.max_blocks_per_seq * block_size);
    if (L < 0 || L > Lcap) {
        if (flag) atomicOr(a.status, PA_DEV_BAD_CONTEXT);
        L = L < 0 ? 0 : Lcap;
    }
    return L;
}

// Work plan: every (sequence, context partition) pair, longest first.  A pair
// covers the partition's blocks; its kv heads are separate work units, handed
// out in list order by an atomic counter.  Full partitions come first, then the
// sequences' last partitions by decreasing length (a counting sort on the block
// count), so the units left at the end of the grid are the short ones.  Order
// within a length is arbitrary and does not change any result.  Each entry also
// carries the (clamped) context length.
//
// With `adaptive` set the partition may grow (doubling from partition_blocks, up to
// the longest context) while the largest unit stays within a quarter of one CTA's
// share of all the work: fewer sequences are split, yet every CTA still gets
// several units to balance with.  The choice is written to plan[2].  The split
// sequences are listed with their context lengths for the merge.
//
// With first_wave > 0 (the host has shown the partition cannot grow) the list
// starts with the pairs (s, partition 0) for s < ceil(first_wave / Hkv), in
// sequence order: the persistent kernel's first CTAs take those units straight from
// their block index while this kernel still runs, and the longest-first order
// covers the other pairs.
__global__ void __launch_bounds__(1024) decode_plan_kernel(const DecodeArgs a, int block_size)
{
    __shared__ int bucket[kMaxPartitionTokens / 16 + 1];
    __shared__ unsigned long long s_tok[32];
    __shared__ int s_max[32];
    __shared__ int s_pb;
    __shared__ int s_nsplit;
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // total and longest context
    unsigned long long tok = 0;
    int lmax = 0;
    for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
        const int L = clamped_context(a, s, block_size, true);
        tok += (unsigned long long)L;
        lmax = max(lmax, L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tok += __shfl_xor_sync(0xffffffffu, tok, o);
        lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    }
    if (lane == 0) {
        s_tok[warp] = tok;
        s_max[warp] = lmax;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long t = 0;
        int m = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            t += s_tok[w];
            m = max(m, s_max[w]);
        }
        int pb = a.partition_blocks;
        if (a.adaptive && a.first_wave == 0) {  // (the first wave fixes the partition at partition_blocks)
            const int max_pb = kMaxPartitionTokens / block_size;
            const double share = (double)t / (double)(a.num_ctas > 0 ? a.num_ctas : 1);  // tokens per CTA, per kv head
            while (2 * pb <= max_pb && pb * block_size < m &&
                   (double)min(2 * pb * block_size, m) * 4.0 <= share)
                pb *= 2;
        }
        s_pb = pb;
        s_nsplit = 0;
        a.plan[2] = (unsigned)pb;
    }
    __syncthreads();
    const int pb = s_pb;
    const int P = pb * block_size;
    const int nfirst = (a.first_wave + a.num_kv_heads - 1) / a.num_kv_heads;  // pairs taken before the plan
    for (int i = threadIdx.x; i <= pb; i += blockDim.x) bucket[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
        const int L = clamped_context(a, s, block_size, false);
        const int np = L > 0 ? (L + P - 1) / P : 1;
        const int last = L > 0 ? (L - (np - 1) * P + block_size - 1) / block_size : 0;
        if (s < nfirst) {
            // pair (s, 0) sits at list position s; only the others are sorted
            a.plan_list[s] = make_uint2((unsigned)s << 11, (unsigned)L);
            atomicAdd(&bucket[np > 1 ? pb : last], -1);
        }
        if (np > 1) {
            atomicAdd(&bucket[pb], np - 1);
            a.split_list[atomicAdd(&s_nsplit, 1)] = make_uint2((unsigned)s, (unsigned)L);
        }
        atomicAdd(&bucket[last], 1);
    }
    __syncthreads();
    if (warp == 0) {
        // exclusive scan over sizes, largest first, after the first-wave pairs:
        // start[sz] = nfirst + pairs of size > sz
        int running = nfirst;
        for (int base = pb; base >= 0; base -= 32) {
            const int sz = base - lane;
            const int c = sz >= 0 ? bucket[sz] : 0;
            int x = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (sz >= 0) bucket[sz] = running + x - c;
            running += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) {
            a.plan[0] = 0u;                 // work counter
            a.plan[4] = 0u;                 // CTAs that stopped taking units (the last one resets both)
            a.plan[1] = (unsigned)running;  // number of (sequence, partition) pairs
            a.plan[3] = (unsigned)s_nsplit; // sequences that need the merge
        }
    }
    __syncthreads();
    for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
        const int L = clamped_context(a, s, block_size, false);
        const int np = L > 0 ? (L + P - 1) / P : 1;
        const int last = L > 0 ? (L - (np - 1) * P + block_size - 1) / block_size : 0;
        for (int p = s < nfirst ? 1 : 0; p < np; ++p) {
            const int sz = p < np - 1 ? pb : last;
            const int pos = atomicAdd(&bucket[sz], 1);
            a.plan_list[pos] = make_uint2(((unsigned)s << 11) | (unsigned)p, (unsigned)L);
        }
    }
}

// Merges the NCW consumer warps' states (m: running max, l: softmax sum, acc:
// unnormalised output, all relative to m) of one (sequence, kv head, partition)
// and writes either the final output row (the sequence fits in one partition) or
// the partition's state to the workspace.  Run by one warp: a lane owns four
// consecutive columns of one query head's row (float4 reads of the states).
//
// Tile j of the unit (j = 0, 1, ...) was consumed by warp (rot + j) % NCW, rot being
// where the unit started in the CTA's stage stream, which depends on the units the
// CTA ran before.  The states are summed in tile-phase order (j mod NCW), not in
// warp order, so the result is the same bits whichever CTA ran the unit and after
// what: the decode is reproducible run to run under the dynamic work counter.
template <typename T, int D, int G, int NCW>
__device__ __forceinline__ void finish_unit_warp(const DecodeArgs& a, const float* mg_m, const float* mg_l,
                                                 const float* mg_acc, int s, int kvh, int part, bool split, int rot,
                                                 int lane)
{
    constexpr int LPG = D / 4;     // lanes per head row
    constexpr int GPP = 32 / LPG;  // head rows per pass
    static_assert(D % 4 == 0 && 32 % LPG == 0, "a warp covers whole head rows");
    const int sub = lane / LPG;
    const int d0 = (lane % LPG) * 4;
#pragma unroll
    for (int g0 = 0; g0 < G; g0 += GPP) {
        const int g = g0 + sub;
        if (g < G) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NCW; ++w) M = fmaxf(M, mg_m[w * G + g]);
            float n0 = 0.f, n1 = 0.f, n2 = 0.f, n3 = 0.f, den = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int j = 0; j < NCW; ++j) {
                    const int w = (rot + j) % NCW;
                    const float mj = mg_m[w * G + g];
                    if (mj != -INFINITY) {
                        const float sc = exp2f(mj - M);
                        const float4 v = *reinterpret_cast<const float4*>(mg_acc + (w * G + g) * D + d0);
                        n0 = fmaf(sc, v.x, n0);
                        n1 = fmaf(sc, v.y, n1);
                        n2 = fmaf(sc, v.z, n2);
                        n3 = fmaf(sc, v.w, n3);
                        den = fmaf(sc, mg_l[w * G + g], den);
                    }
                }
            }
            const int h = kvh * G + g;
            if (!split) {
                T* o = static_cast<T*>(a.out) + ((size_t)s * a.num_heads + h) * D + d0;
                const bool any = den > 0.f;
                const float r0 = any ? n0 / den : 0.f, r1 = any ? n1 / den : 0.f;
                const float r2 = any ? n2 / den : 0.f, r3 = any ? n3 / den : 0.f;
                if constexpr (sizeof(T) == 4) {
                    *reinterpret_cast<float4*>(o) = make_float4(r0, r1, r2, r3);
                } else {
                    const __nv_bfloat162 lo = __floats2bfloat162_rn(r0, r1);
                    const __nv_bfloat162 hi = __floats2bfloat162_rn(r2, r3);
                    uint2 pk;
                    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
                    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
                    *reinterpret_cast<uint2*>(o) = pk;
                }
            } else {
                const size_t row = ((size_t)s * a.num_heads + h) * a.num_partitions + part;
                *reinterpret_cast<float4*>(a.ws_acc + row * D + d0) = make_float4(n0, n1, n2, n3);
                if (d0 == 0) {
                    a.ws_ml[row * 2] = M;
                    a.ws_ml[row * 2 + 1] = den;
                }
            }
        }
    }
}

// Log-sum-exp merge of the partitions of the split sequences the plan listed:
// M = max_p m_p, out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p, per
// (sequence, query head) row.  `nwr` warps share a row (1, 2 or 4; a CTA of four
// warps holds 4 / nwr rows at a time, CTAs striding over the rows).  A lane owns
// D/32 consecutive columns.  The partitions go in chunks of 8, chunk c to warp
// c % nwr of the row, whose eight column loads are all in flight together.  The
// warps' sums are added in warp order, so a row's bits do not depend on the CTA that
// merges it.
//
// The kernel is latency-bound, so its loads are arranged to wait on as little as
// possible.  The plan lists each split sequence together with its context length,
// and the first chunk's columns are requested together with the partition maxima.
// A row then costs two dependent round trips to memory: the list entry, then the
// partition states.
template <typename T, int D>
__global__ void __launch_bounds__(128, 8) decode_merge_kernel(const DecodeArgs a, int block_size, int nwr)
{
    constexpr int EPL = D / 32;
    constexpr int CH = 8;
    __shared__ __align__(16) float s_num[4][D];
    __shared__ float s_den[4];
    pdl_wait_primary();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rpc = 4 / nwr;  // rows per CTA at a time
    const int slot = warp / nwr, sub = warp % nwr;
    const int H = a.num_heads;
    const unsigned* plan = a.plan;
    const int P = (int)__ldg(plan + 2) * block_size;
    const int rows = (int)__ldg(plan + 3) * H;
    // the first row's list entry, requested with the counts above (the index stays
    // inside the list, which has a slot per sequence, whatever the count turns out to be)
    uint2 e = __ldg(a.split_list + min((int)blockIdx.x * rpc + slot, a.num_seqs * H - 1) / H);
    for (int r0 = blockIdx.x * rpc; r0 < rows; r0 += gridDim.x * rpc) {
        const int r = r0 + slot;
        float num[EPL];
#pragma unroll
        for (int k = 0; k < EPL; ++k) num[k] = 0.f;
        float den = 0.f;
        if (r < rows) {
            if (r0 != (int)blockIdx.x * rpc) e = __ldg(a.split_list + r / H);
            const int L = (int)e.y;
            const int np = (L + P - 1) / P;
            const size_t row0 = ((size_t)e.x * H + r % H) * a.num_partitions;
            const float2* ml = reinterpret_cast<const float2*>(a.ws_ml) + row0;
            const float* acc = a.ws_acc + row0 * D + lane * EPL;
            float x[CH][EPL];
            auto load_chunk = [&](int c) {
#pragma unroll
                for (int u = 0; u < CH; ++u) {
                    // partitions past np repeat the last one; their weight is 0
                    const float* src = acc + (size_t)min(c * CH + u, np - 1) * D;
                    if constexpr (EPL == 4) {
                        const float4 v = __ldg(reinterpret_cast<const float4*>(src));
                        x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
                    } else {
                        const float2 v = __ldg(reinterpret_cast<const float2*>(src));
                        x[u][0] = v.x; x[u][1] = v.y;
                    }
                }
            };
            int c = sub;
            if (c * CH < np) load_chunk(c);
            float M = -INFINITY;
            for (int p = lane; p < np; p += 32) M = fmaxf(M, __ldg(&ml[p].x));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            for (; c * CH < np; c += nwr) {
                if (c != sub) load_chunk(c);
                // lane u < 8 holds the weight of partition c * 8 + u
                const int pw = c * CH + (lane & (CH - 1));
                float w = 0.f;
                if (lane < CH && pw < np) {
                    const float2 v = __ldg(ml + pw);
                    w = v.x == -INFINITY ? 0.f : exp2f(v.x - M);
                    den = fmaf(w, v.y, den);
                }
#pragma unroll
                for (int u = 0; u < CH; ++u) {
                    const float wu = __shfl_sync(0xffffffffu, w, u);
#pragma unroll
                    for (int k = 0; k < EPL; ++k) num[k] = fmaf(wu, x[u][k], num[k]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        }
        if (nwr > 1) {
#pragma unroll
            for (int k = 0; k < EPL; ++k) s_num[warp][lane * EPL + k] = num[k];
            if (lane == 0) s_den[warp] = den;
            __syncthreads();
            if (sub == 0) {
                for (int j = 1; j < nwr; ++j) {
#pragma unroll
                    for (int k = 0; k < EPL; ++k) num[k] += s_num[warp + j][lane * EPL + k];
                    den += s_den[warp + j];
                }
            }
            __syncthreads();
        }
        if (r < rows && sub == 0) {
            const float inv = den > 0.f ? 1.f / den : 0.f;
            T* o = static_cast<T*>(a.out) + ((size_t)e.x * H + r % H) * D + lane * EPL;
#pragma unroll
            for (int k = 0; k < EPL; ++k) o[k] = from_f32<T>(num[k] * inv);
        }
    }
}

// Launches a kernel with programmatic dependent launch: its CTAs may be scheduled
// while the previous kernel in the stream drains; they wait (griddepcontrol.wait)
// before touching that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename T, int D>
cudaError_t launch_merge(const DecodeArgs& a, int block_size, cudaStream_t stream)
{
    // one warp per row while a row has at most one chunk of 8 partitions, two for two
    // chunks, else four; up to eight CTAs per SM, striding over the rows of the split sequences
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int nwr = a.num_partitions <= 8 ? 1 : (a.num_partitions <= 16 ? 2 : 4);
    const long rpc = 4 / nwr;
    const long ctas = ((long)a.num_seqs * a.num_heads + rpc - 1) / rpc;
    const unsigned grid = (unsigned)(ctas < 8L * sms ? ctas : 8L * sms);
    return launch_pdl(decode_merge_kernel<T, D>, dim3(grid), dim3(128), 0, stream, a, block_size, nwr);
}

}  // namespace
}  // namespace pa
