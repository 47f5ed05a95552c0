// Pieces of the paged decode path shared by its two consumers (CUDA cores and
// tensor cores): vector loads, the longest-first work plan, the per-partition
// epilogue that merges the consumer warps' softmax states, and the log-sum-exp
// merge of a sequence's context partitions at the tail of the grid.
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
            // the sequence's merge counters start at zero (every run leaves them there too)
            for (int k = 0; k < a.num_kv_heads; ++k) {
                a.ready[(size_t)s * a.num_kv_heads + k] = 0u;
                a.ready[((size_t)a.num_seqs + s) * a.num_kv_heads + k] = 0u;
            }
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
            a.plan[5] = 0u;                 // merge-row counter
            a.plan[6] = 0u;                 // consumer warps done merging (the last one resets 5, 6, 7)
            a.plan[7] = 0u;                 // CTAs started
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

// Log-sum-exp merge of one (sequence, query head) row of a split sequence:
// M = max_p m_p, out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p over its np
// partitions, written to out.  Run by one warp; a lane owns D/32 consecutive columns.
// The partitions go in chunks of 8 whose column loads are all in flight together,
// and chunk 0's loads are issued before the maxima are reduced.  The sums run in
// partition order, so a row's bits do not depend on the warp that merges it.  The
// partition states are read from L2 (another CTA wrote them).
template <typename T, int D>
__device__ __forceinline__ void merge_split_row(const DecodeArgs& a, int s, int h, int np, int lane)
{
    constexpr int EPL = D / 32;
    constexpr int CH = 8;
    const size_t row0 = ((size_t)s * a.num_heads + h) * a.num_partitions;
    const float2* ml = reinterpret_cast<const float2*>(a.ws_ml) + row0;
    const float* acc = a.ws_acc + row0 * D + lane * EPL;
    float x[CH][EPL];
    auto load_chunk = [&](int c) {
#pragma unroll
        for (int u = 0; u < CH; ++u) {
            // partitions past np repeat the last one; their weight is 0
            const float* src = acc + (size_t)min(c * CH + u, np - 1) * D;
            if constexpr (EPL == 4) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
                x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
            } else {
                const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
                x[u][0] = v.x; x[u][1] = v.y;
            }
        }
    };
    load_chunk(0);
    float M = -INFINITY;
    for (int p = lane; p < np; p += 32) M = fmaxf(M, __ldcg(&ml[p].x));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float num[EPL];
#pragma unroll
    for (int k = 0; k < EPL; ++k) num[k] = 0.f;
    float den = 0.f;
    for (int c = 0; c * CH < np; ++c) {
        if (c > 0) load_chunk(c);
        // lane u < 8 holds the weight of partition c * 8 + u
        const int pw = c * CH + (lane & (CH - 1));
        float w = 0.f;
        if (lane < CH && pw < np) {
            const float2 v = __ldcg(ml + pw);
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
    const float inv = den > 0.f ? 1.f / den : 0.f;
    T* o = static_cast<T*>(a.out) + ((size_t)s * a.num_heads + h) * D + lane * EPL;
#pragma unroll
    for (int k = 0; k < EPL; ++k) o[k] = from_f32<T>(num[k] * inv);
}

// The merge of the split sequences' partitions, run by the persistent kernel's
// consumer warps once they have no more units (the tail of the grid, where CTAs would
// otherwise idle), instead of a separate kernel after the whole grid has drained.
// Rows (split sequence, query head) are claimed from a counter in list order; a row
// waits until all partitions of its (sequence, kv head) are finished (a release count
// kept by the warps that wrote the partition states), merges them and writes out.
//
// A warp waits on other CTAs only when every CTA of the grid has started: then every
// unit not yet finished belongs to a running CTA, which never waits on another, so
// each wait ends.  A warp that sees the grid not yet fully started merges nothing
// (the CTAs still to start will, the last of them certainly).  The last consumer warp
// of the grid to finish resets the counters, so a plan serves the next run as is.
// `ok` is false when this warp gave up earlier: it then only counts itself out.
template <typename T, int D, int G>
__device__ __forceinline__ void tail_merge_warp(const DecodeArgs& a, int block_size, bool ok, int lane,
                                                unsigned total_warps)
{
    const unsigned H = (unsigned)a.num_heads;
    const unsigned Hkv = (unsigned)a.num_kv_heads;
    unsigned go = 0;
    if (lane == 0 && ok) go = ld_acquire(a.plan + 7) >= gridDim.x ? 1u : 0u;
    go = __shfl_sync(0xffffffffu, go, 0);
    if (go) {
        const unsigned nrows = __ldcg(a.plan + 3) * H;
        const int P = (int)__ldcg(a.plan + 2) * block_size;
        for (;;) {
            unsigned r = 0;
            if (lane == 0) r = atomicAdd(a.plan + 5, 1u);
            r = __shfl_sync(0xffffffffu, r, 0);
            if (r >= nrows) break;
            const uint2 e = __ldcg(a.split_list + r / H);
            const int s = (int)e.x, h = (int)(r % H), L = (int)e.y;
            const int np = (L + P - 1) / P;
            const size_t key = (size_t)s * Hkv + (unsigned)h / G;
            unsigned done = 1;
            if (lane == 0) done = wait_count_bounded(a.ready + key, (unsigned)np) ? 1u : 0u;
            done = __shfl_sync(0xffffffffu, done, 0);
            if (!done) {
                if (lane == 0) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                break;
            }
            merge_split_row<T, D>(a, s, h, np, lane);
            if (lane == 0) {
                // the kv head's last row merged: its counters go back to zero for the next run
                unsigned int* merged = a.ready + (size_t)a.num_seqs * Hkv + key;
                if (atomicAdd(merged, 1u) == (unsigned)G - 1) {
                    a.ready[key] = 0u;
                    *merged = 0u;
                }
            }
        }
    }
    if (lane == 0 && atomicAdd(a.plan + 6, 1u) == total_warps - 1) {
        a.plan[5] = 0u;
        a.plan[6] = 0u;
        a.plan[7] = 0u;
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

}  // namespace
}  // namespace pa
