// CUDA-core consumer of the paged decode kernel: fp32 inputs, and bf16 with one
// query head per kv head.  One warp processes one physical block at a time and
// keeps its own online-softmax state ("PagedAttention and vLLM Architecture",
// section 2: dot q with every key of the gathered block, online softmax across
// blocks, fused product with the block's V rows).
//
// Every lane reads 16-byte vectors of the K and V rows (LPR lanes cover one row,
// RPW rows per warp step).  The G x (rows) partial dot products of a lane are
// summed across the LPR lanes of its row with a transposing butterfly: each step
// halves the values a lane holds, so the sum of NV values over LPR lanes takes
// log2(LPR) steps and about NV shuffles instead of NV * log2(LPR).  The softmax
// weights go back to all lanes through a small per-warp shared buffer.
#pragma once

#include "pa_decode_common.cuh"

namespace pa {
namespace {

// Sums N per-lane values across the lanes of each group of 2*OFF (xor offsets
// OFF .. 1), halving the values a lane holds at each step while N >= 2.  Lane c
// of a group of LPR lanes ends with max(1, N/LPR) full sums, value indices
// starting at c*N/LPR.
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

template <typename T_, int D_, int B_, int G_>
struct FmaConsumer {
    using T = T_;
    static constexpr int D = D_, B = B_, G = G_;
    static constexpr bool kTensorLoads = false;            // whole tiles by 1-D bulk copies
    static constexpr int kElt = sizeof(T);
    static constexpr int EPL = 16 / kElt;                  // elements per lane vector
    static constexpr int LPR = D * kElt / 16;              // lanes covering one token row
    static constexpr int RPW = 32 / LPR;                   // rows a warp reads per step
    static constexpr int TPL = B / RPW;                    // row steps per block
    static constexpr int TPC = cmax(1, cmin(TPL, 32 / G)); // row steps per softmax chunk
    static constexpr int NCH = TPL / TPC;                  // chunks per block
    static constexpr int NV = G * TPC;                     // partial logits per lane per chunk
    static constexpr int NVO = NV >= LPR ? NV / LPR : 1;   // full logits a lane holds after the butterfly
    static constexpr int DUP = NV >= LPR ? 1 : LPR / NV;   // lanes holding the same logit
    static constexpr int LPH = LPR / G;                    // lanes of a row group sharing one head
    static constexpr int SCRATCH_FLOATS = RPW * NV + G;    // per warp: weights [RPW][TPC][G], new maxima [G]

    static_assert(16 % kElt == 0 && D % EPL == 0, "vector width");
    static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "row lanes");
    static_assert(B % RPW == 0 && TPL % TPC == 0, "block split");
    static_assert(G <= LPR, "group larger than a row's lanes");

    float qf[G][EPL];     // q (pre-scaled to base-2 logits), this lane's columns
    float m_run[G];       // running max per head (same in every lane)
    float acc[G][EPL];    // unnormalised output, this lane's columns, row group r
    float l_own;          // running sum of this lane's logits (head g_own)
    float m_own;          // running max of head g_own
    int lane, c, r, g_own, idx0;
    float* p_w;
    float* m_w;

    __device__ __forceinline__ void init(float* scratch, int lane_)
    {
        lane = lane_;
        c = lane % LPR;
        r = lane / LPR;
        g_own = (c * G) / LPR;
        idx0 = (c * NV) / LPR;
        p_w = scratch;
        m_w = scratch + RPW * NV;
    }

    __device__ __forceinline__ void begin_unit(const T* q_smem, float scale_log2)
    {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            load16_f32<T>(q_smem + g * D + c * EPL, qf[g]);
#pragma unroll
            for (int e = 0; e < EPL; ++e) qf[g][e] *= scale_log2;
            m_run[g] = -INFINITY;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
        }
        l_own = 0.f;
        m_own = -INFINITY;
    }

    // One physical block: K tile kt and V tile vt ([B][D] in shared memory); rows
    // nvalid.. are past the context and contribute nothing.
    __device__ __forceinline__ void block(const unsigned char* kt_, unsigned char* vt_, int nvalid)
    {
        const T* kt = reinterpret_cast<const T*>(kt_);
        const T* vt = reinterpret_cast<const T*>(vt_);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
            // q . K for this chunk's rows: v[g*TPC + t], row j = (ch*TPC + t)*RPW + r
            float v[NV];
#pragma unroll
            for (int t = 0; t < TPC; ++t) {
                const int j = (ch * TPC + t) * RPW + r;
                float kf[EPL];
                load16_f32<T>(kt + j * D + c * EPL, kf);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float sum = 0.f;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) sum = fmaf(qf[g][e], kf[e], sum);
                    v[g * TPC + t] = sum;
                }
            }
            Butterfly<NV, LPR / 2>::run(v, lane);

            // This lane now holds logits idx0 .. idx0+NVO-1, all of head g_own.
            float cmax_ = -INFINITY;
#pragma unroll
            for (int k = 0; k < NVO; ++k) {
                const int t = (idx0 + k) % TPC;
                const int j = (ch * TPC + t) * RPW + r;
                if (j >= nvalid) v[k] = -INFINITY;
                cmax_ = fmaxf(cmax_, v[k]);
            }
            cmax_ = head_allreduce<LPH, LPR, true>(cmax_);
            const float m_new = fmaxf(m_own, cmax_);
            const float alpha_own = exp2f(m_own - m_new);
            m_own = m_new;
            float psum = 0.f;
#pragma unroll
            for (int k = 0; k < NVO; ++k) {
                const float p = exp2f(v[k] - m_new);
                psum += p;
                const int t = (idx0 + k) % TPC;
                p_w[(r * TPC + t) * G + g_own] = p;
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
                    for (int e = 0; e < EPL; ++e) acc[g][e] *= alpha;
                    m_run[g] = mg;
                }
            }
            // P . V for this chunk's rows
#pragma unroll
            for (int t = 0; t < TPC; ++t) {
                const int j = (ch * TPC + t) * RPW + r;
                if (j < nvalid) {
                    float vf[EPL];
                    load16_f32<T>(vt + j * D + c * EPL, vf);
                    float pg[G];
                    const float* pp = p_w + (r * TPC + t) * G;
#pragma unroll
                    for (int g = 0; g < G; ++g) pg[g] = pp[g];
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(pg[g], vf[e], acc[g][e]);
                }
            }
            __syncwarp();
        }
    }

    // Writes this warp's (m, l, acc) into the merge area.
    __device__ __forceinline__ void end_unit(float* mg_m, float* mg_l, float* mg_acc, int warp)
    {
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
        const float l = head_allreduce<LPH, LPR, false>(l_own) * (1.0f / DUP);
        if (lane == 0)
#pragma unroll
            for (int g = 0; g < G; ++g) mg_m[warp * G + g] = m_run[g];
        if (r == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < EPL; ++e) mg_acc[(warp * G + g) * D + c * EPL + e] = acc[g][e];
        }
        if (c % LPH == 0 && r == 0) mg_l[warp * G + g_own] = l;
    }
};

}  // namespace
}  // namespace pa
