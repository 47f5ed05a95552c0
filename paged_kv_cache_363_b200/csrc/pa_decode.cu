// Paged decode attention for sm_100a.
//
// What it computes ("PagedAttention and vLLM Architecture", section 2, "PagedAttention
// Attention CUDA Kernel Mechanics"): for each sequence's single new query, walk the
// physical blocks named by the block table in logical order, dot q with every key of
// each gathered block, keep an online softmax (running max and sum) across blocks and
// fold the weighted V rows of the same blocks into the output in the same pass.
// Token i of a sequence lives in physical block T[i / B] at offset i % B
// ("PagedAttention Paper Breakdown", section 2, Address Translation Formula).
//
// B200 design:
//  * One CTA per (kv head, sequence, context partition).  All query heads of the
//    kv head's group are packed into the CTA, so each K/V byte leaves HBM once.
//  * A physical block's K tile (and its V tile) for one kv head is one contiguous run
//    of B*D elements in the [num_blocks][kv_heads][B][D] pool, so a single producer
//    thread streams whole tiles with 1-D bulk copies (the TMA engine, no tensor map,
//    no multicast) into a ring of shared-memory stages guarded by mbarriers.
//  * Four consumer warps take alternate blocks, each with its own online-softmax
//    state; the states are merged once per partition.  Inside a warp every lane
//    reads 16-byte vectors; the B x G logits are summed across the lanes of a row
//    with a transposing butterfly (each step halves the values a lane holds), and the
//    softmax weights are shared through a small per-warp shared buffer.
//  * Sequences longer than one partition leave (max, sum, unnormalised output) per
//    partition in the workspace; a second kernel merges them by log-sum-exp.  That
//    kernel is launched with programmatic dependent launch so its launch overlaps the
//    first kernel's tail.
//  * Logits are kept in base-2 units (q pre-scaled by scale*log2 e) and exponentials
//    use exp2f, the reformulation of online softmax by Milakov & Gimelshein (2018).
//  * Every wait is bounded; bad block indices or context lengths raise a status bit
//    and are clamped instead of being dereferenced.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cfloat>
#include <cstdint>

#include "pa_decode_common.cuh"
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {

namespace {

template <typename T, int D, int B, int G>
struct Cfg {
    static constexpr int kElt = sizeof(T);
    static constexpr int EPL = 16 / kElt;                 // elements per lane vector
    static constexpr int LPR = D * kElt / 16;             // lanes covering one token row
    static constexpr int RPW = 32 / LPR;                  // rows a warp reads per step
    static constexpr int TPL = B / RPW;                   // row steps per block
    static constexpr int TPC = cmax(1, cmin(TPL, 32 / G));  // row steps per softmax chunk
    static constexpr int NCH = TPL / TPC;                 // chunks per block
    static constexpr int NV = G * TPC;                    // partial logits per lane per chunk
    static constexpr int NVO = NV >= LPR ? NV / LPR : 1;  // full logits a lane holds after the butterfly
    static constexpr int DUP = NV >= LPR ? 1 : LPR / NV;  // lanes holding the same logit
    static constexpr int LPH = LPR / G;                   // lanes of a row group sharing one head
    static constexpr int TILE = B * D;                    // elements of one K (or V) tile
    static constexpr int TILE_BYTES = TILE * kElt;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int NCW = 4;                         // consumer warps
    // Stage i % NSTAGES holds block i and warp i % NCW consumes it.  With NSTAGES a
    // multiple of NCW the warp that waits for a stage's n-th fill also consumed its
    // (n-1)-th, so the one-bit phase parity of the wait can never be stale.
    static constexpr int NSTAGES = cmax(NCW, cmin(8, 65536 / STAGE_BYTES));
    static constexpr int THREADS = (NCW + 1) * 32;
    static constexpr int MAX_PBLK = kMaxPartitionTokens / 16;
    // shared-memory carve-up (bytes)
    static constexpr int OFF_BAR = NSTAGES * STAGE_BYTES;
    static constexpr int OFF_TABLE = OFF_BAR + 2 * NSTAGES * 8;
    static constexpr int OFF_P = OFF_TABLE + MAX_PBLK * 4;
    static constexpr int P_FLOATS = NCW * RPW * NV;       // per warp: [RPW][TPC][G]
    static constexpr int OFF_M = OFF_P + P_FLOATS * 4;
    static constexpr int OFF_ABORT = OFF_M + NCW * G * 4;
    static constexpr int SMEM = OFF_ABORT + 16;
    // merge area (aliases the stages once the pipeline has drained)
    static constexpr int MERGE_BYTES = NCW * G * (D + 2) * 4;

    static_assert(16 % kElt == 0 && D % EPL == 0, "vector width");
    static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "row lanes");
    static_assert(B % RPW == 0 && TPL % TPC == 0, "block split");
    static_assert(G <= LPR, "group larger than a row's lanes");
    static_assert(MERGE_BYTES <= OFF_BAR, "merge area must fit in the stage ring");
    static_assert(TILE_BYTES % 16 == 0, "bulk copy size");
    static_assert(NSTAGES % NCW == 0, "stage ring must be a multiple of the consumer warps");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// Sums N per-lane values across the LPR lanes of each row group (xor offsets
// LPR/2 .. 1), halving the values a lane holds at each step while N >= 2.  Lane c
// of a group ends with max(1, N/LPR) full sums, value indices starting at c*N/LPR.
template <int N, int OFF>
struct Butterfly {
    static __device__ __forceinline__ void run(float* v, int lane)
    {
        if constexpr (OFF >= 1) {
            if constexpr (N >= 2) {
                const bool up = (lane & OFF) != 0;
#pragma unroll
                for (int i = 0; i < N / 2; ++i) {
                    const float lo = v[i];
                    const float hi = v[i + N / 2];
                    const float send = up ? lo : hi;
                    const float keep = up ? hi : lo;
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
                }
                Butterfly<N / 2, OFF / 2>::run(v, lane);
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
                Butterfly<1, OFF / 2>::run(v, lane);
            }
        }
    }
};

// Max (or sum) over the lanes that share a head: the LPH lanes inside a row group
// and the same lanes of every row group.
template <int LPH, int LPR, bool MAX>
__device__ __forceinline__ float head_allreduce(float x)
{
#pragma unroll
    for (int o = 1; o < LPH; o <<= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, x, o);
        x = MAX ? fmaxf(x, y) : x + y;
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, x, o);
        x = MAX ? fmaxf(x, y) : x + y;
    }
    return x;
}

// Three CTAs per SM (about 200 KB of stages in flight); a group of 8 heads needs
// more registers per thread and runs two.
template <typename T, int D, int B, int G>
__global__ void __launch_bounds__(Cfg<T, D, B, G>::THREADS, (G >= 8 ? 2 : 3))
    decode_partition_kernel(const DecodeArgs a)
{
    using C = Cfg<T, D, B, G>;
    extern __shared__ __align__(128) unsigned char smem[];
    T* stages = reinterpret_cast<T*>(smem);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty_bar = full_bar + C::NSTAGES;
    int* s_table = reinterpret_cast<int*>(smem + C::OFF_TABLE);
    float* s_p = reinterpret_cast<float*>(smem + C::OFF_P);
    float* s_m = reinterpret_cast<float*>(smem + C::OFF_M);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);

    const int kvh = blockIdx.x;
    const int s = blockIdx.y;
    const int part = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Sequences that fit in fewer partitions exit at once; the exit also lets the
    // merge kernel (programmatic dependent launch) start once every CTA got here.
    pdl_launch_dependents();

    int L = __ldg(a.context_lens + s);
    const int Lcap = min(a.max_context_len, a.max_blocks_per_seq * B);
    if (L < 0 || L > Lcap) {
        if (threadIdx.x == 0 && part == 0 && kvh == 0) atomicOr(a.status, PA_DEV_BAD_CONTEXT);
        L = L < 0 ? 0 : Lcap;
    }
    const int nblk_seq = (L + B - 1) / B;
    const int pb = a.partition_blocks;
    const int b0 = part * pb;
    if (part > 0 && b0 >= nblk_seq) return;
    const int nblk = max(0, min(pb, nblk_seq - b0));
    const bool split = nblk_seq > pb;

    for (int i = threadIdx.x; i < nblk; i += C::THREADS)
        s_table[i] = __ldg(a.block_tables + (size_t)s * a.max_blocks_per_seq + b0 + i);
    if (threadIdx.x == 0) {
#pragma unroll
        for (int st = 0; st < C::NSTAGES; ++st) {
            mbar_init(&full_bar[st], 1);
            mbar_init(&empty_bar[st], 1);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const float NEG_INF = -INFINITY;
    const int c = lane % C::LPR;  // 16-byte column chunk of the row this lane reads
    const int r = lane / C::LPR;  // row group
    float m_run[G];               // running max per head (same in every lane)
    float acc[G][C::EPL];         // unnormalised output, this lane's columns, row group r
    float l_own = 0.f;            // running sum of this lane's logits (head g_own)
    float m_own = NEG_INF;        // running max of head g_own
    const int g_own = (c * G) / C::LPR;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m_run[g] = NEG_INF;
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) acc[g][e] = 0.f;
    }

    if (warp == C::NCW) {
        // ---------------- producer: one thread streams K/V tiles into the ring
        if (lane == 0) {
            const T* kc = static_cast<const T*>(a.k_cache);
            const T* vc = static_cast<const T*>(a.v_cache);
            const uint64_t policy = policy_evict_first();
            int issued = 0;
            bool ok = true;
            for (int i = 0; i < nblk; ++i) {
                const int st = i % C::NSTAGES;
                if (i >= C::NSTAGES &&
                    !mbar_wait_bounded(&empty_bar[st], ((i / C::NSTAGES) & 1) ^ 1, s_abort)) {
                    ok = false;
                    break;
                }
                int phys = s_table[i];
                if ((unsigned)phys >= (unsigned)a.num_blocks) {
                    atomicOr(a.status, PA_DEV_BAD_BLOCK);
                    phys = 0;
                }
                const size_t off = ((size_t)phys * a.num_kv_heads + kvh) * C::TILE;
                T* dk = stages + (size_t)st * 2 * C::TILE;
                mbar_arrive_expect_tx(&full_bar[st], 2 * C::TILE_BYTES);
                bulk_g2s_hint(dk, kc + off, C::TILE_BYTES, &full_bar[st], policy);
                bulk_g2s_hint(dk + C::TILE, vc + off, C::TILE_BYTES, &full_bar[st], policy);
                ++issued;
            }
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *s_abort = 1;
            }
            // Drain: no bulk copy may still be landing in shared memory at exit.
            volatile int never = 0;
            for (int i = max(0, issued - C::NSTAGES); i < issued; ++i)
                if (!mbar_wait_bounded(&full_bar[i % C::NSTAGES], (i / C::NSTAGES) & 1, &never))
                    atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else {
        // ---------------- consumers
        float qf[G][C::EPL];
        {
            const T* qp = static_cast<const T*>(a.q) + ((size_t)s * a.num_heads + (size_t)kvh * G) * D;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                load16_f32<T>(qp + g * D + c * C::EPL, qf[g]);
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) qf[g][e] *= a.scale_log2;
            }
        }
        float* p_w = s_p + warp * (C::RPW * C::NV);  // [RPW][TPC][G]
        float* m_w = s_m + warp * G;
        const int idx0 = (c * C::NV) / C::LPR;       // first logit index this lane holds

        for (int i = warp; i < nblk; i += C::NCW) {
            const int st = i % C::NSTAGES;
            if (!mbar_wait_bounded(&full_bar[st], (i / C::NSTAGES) & 1, s_abort)) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *s_abort = 1;
                break;
            }
            const T* kt = stages + (size_t)st * 2 * C::TILE;
            const T* vt = kt + C::TILE;
            const int nvalid = min(B, L - (b0 + i) * B);

#pragma unroll
            for (int ch = 0; ch < C::NCH; ++ch) {
                // q . K for this chunk's rows: v[g*TPC + t], row j = (ch*TPC + t)*RPW + r
                float v[C::NV];
#pragma unroll
                for (int t = 0; t < C::TPC; ++t) {
                    const int j = (ch * C::TPC + t) * C::RPW + r;
                    float kf[C::EPL];
                    load16_f32<T>(kt + j * D + c * C::EPL, kf);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float sum = 0.f;
#pragma unroll
                        for (int e = 0; e < C::EPL; ++e) sum = fmaf(qf[g][e], kf[e], sum);
                        v[g * C::TPC + t] = sum;
                    }
                }
                Butterfly<C::NV, C::LPR / 2>::run(v, lane);

                // This lane now holds logits idx0 .. idx0+NVO-1, all of head g_own.
                float cmax_ = NEG_INF;
#pragma unroll
                for (int k = 0; k < C::NVO; ++k) {
                    const int t = (idx0 + k) % C::TPC;
                    const int j = (ch * C::TPC + t) * C::RPW + r;
                    if (j >= nvalid) v[k] = NEG_INF;
                    cmax_ = fmaxf(cmax_, v[k]);
                }
                cmax_ = head_allreduce<C::LPH, C::LPR, true>(cmax_);
                const float m_new = fmaxf(m_own, cmax_);
                const float alpha_own = exp2f(m_own - m_new);
                m_own = m_new;
                float psum = 0.f;
#pragma unroll
                for (int k = 0; k < C::NVO; ++k) {
                    const float p = exp2f(v[k] - m_new);
                    psum += p;
                    const int t = (idx0 + k) % C::TPC;
                    p_w[(r * C::TPC + t) * G + g_own] = p;
                }
                l_own = l_own * alpha_own + psum;
                m_w[g_own] = m_new;
                __syncwarp();

                // rescale the accumulators of heads whose max moved
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float mg = m_w[g];
                    if (mg != m_run[g]) {
                        const float alpha = exp2f(m_run[g] - mg);
#pragma unroll
                        for (int e = 0; e < C::EPL; ++e) acc[g][e] *= alpha;
                        m_run[g] = mg;
                    }
                }
                // P . V for this chunk's rows
#pragma unroll
                for (int t = 0; t < C::TPC; ++t) {
                    const int j = (ch * C::TPC + t) * C::RPW + r;
                    if (j < nvalid) {
                        float vf[C::EPL];
                        load16_f32<T>(vt + j * D + c * C::EPL, vf);
                        float pg[G];
                        const float* pp = p_w + (r * C::TPC + t) * G;
#pragma unroll
                        for (int g = 0; g < G; ++g) pg[g] = pp[g];
#pragma unroll
                        for (int g = 0; g < G; ++g)
#pragma unroll
                            for (int e = 0; e < C::EPL; ++e) acc[g][e] = fmaf(pg[g], vf[e], acc[g][e]);
                    }
                }
                __syncwarp();
            }
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }

        // fold the row groups together (same columns, different rows)
#pragma unroll
        for (int o = C::LPR; o < 32; o <<= 1)
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
        l_own = head_allreduce<C::LPH, C::LPR, false>(l_own) * (1.0f / C::DUP);
    }

    __syncthreads();  // the stage ring is free from here on: reuse it for the merge

    float* mg_m = reinterpret_cast<float*>(smem);       // [NCW][G]
    float* mg_l = mg_m + C::NCW * G;                    // [NCW][G]
    float* mg_acc = mg_l + C::NCW * G;                  // [NCW][G][D]
    if (warp < C::NCW) {
        if (lane == 0)
#pragma unroll
            for (int g = 0; g < G; ++g) mg_m[warp * G + g] = m_run[g];
        if (r == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) mg_acc[(warp * G + g) * D + c * C::EPL + e] = acc[g][e];
        }
        if (c % C::LPH == 0 && r == 0) mg_l[warp * G + g_own] = l_own;
    }
    __syncthreads();

    finish_partition<T, D, G, C::NCW, C::THREADS>(a, mg_m, mg_l, mg_acc, s, kvh, part, split);
}

template <typename T, int D, int B, int G>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t stream)
{
    using C = Cfg<T, D, B, G>;
    // The shared-memory opt-in is a per-device function attribute: set it once per device.
    static std::atomic<uint64_t> attr_set{0};
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) return e0;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(decode_partition_kernel<T, D, B, G>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit);
    }
    dim3 grid(a.num_kv_heads, a.num_seqs, a.num_partitions);
    decode_partition_kernel<T, D, B, G><<<grid, C::THREADS, C::SMEM, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.num_partitions <= 1) return e;

    return launch_merge<T, D>(a, B, stream);
}

template <typename T, int D, int B>
cudaError_t dispatch_group(const DecodeArgs& a, int group, cudaStream_t stream)
{
    switch (group) {
        case 1: return launch_typed<T, D, B, 1>(a, stream);
        case 2: return launch_typed<T, D, B, 2>(a, stream);
        case 4: return launch_typed<T, D, B, 4>(a, stream);
        case 8: return launch_typed<T, D, B, 8>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, int D>
cudaError_t dispatch_block(const DecodeArgs& a, int block_size, int group, cudaStream_t stream)
{
    switch (block_size) {
        case 16: return dispatch_group<T, D, 16>(a, group, stream);
        case 32: return dispatch_group<T, D, 32>(a, group, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t dispatch_dim(const DecodeArgs& a, int head_dim, int block_size, int group, cudaStream_t stream)
{
    switch (head_dim) {
        case 64: return dispatch_block<T, 64>(a, block_size, group, stream);
        case 128: return dispatch_block<T, 128>(a, block_size, group, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, pa_dtype dtype, int head_dim, int block_size, int group,
                          cudaStream_t stream)
{
    if (decode_uses_tensor_cores(dtype, head_dim, group)) return launch_decode_mma(a, head_dim, block_size, group, stream);
    if (dtype == PA_DTYPE_F32) return dispatch_dim<float>(a, head_dim, block_size, group, stream);
    return dispatch_dim<__nv_bfloat16>(a, head_dim, block_size, group, stream);
}

}  // namespace pa
