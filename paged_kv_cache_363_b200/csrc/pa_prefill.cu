// Chunked prefill attention over the paged KV cache on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory), for sm_100a.
//
// What it computes: the multi-token case of the decode attention.  Sequence s holds
// L_s tokens in the pools (its new tokens already appended, as for decode), of which
// the last n_s are queries; query i sits at position p = L_s - n_s + i and attends to
// tokens 0..p through the block table ("PagedAttention and vLLM Architecture",
// section 3: the prompt's blocks are assigned when it is processed; "PagedAttention
// Paper Breakdown", section 2: token t lives at slot T[t / B] * B + t % B).
//
// A CTA owns one (sequence, kv head) and two query tiles A and B of 128 rows each.  A
// tile's rows are T query tokens x G query heads of the kv head's group (T = 128 / G),
// so every K/V byte the CTA loads serves both tiles and all G heads.  It walks the keys
// in tiles of 128 tokens:
//   - warp 16 stages both Q tiles once and each K and V tile by TMA, one 16-row box per
//     (16-token run of a physical block, 64 columns), 128-byte swizzle, K and V in two
//     32 KB stages each; lane i looks up and issues box i of the tile;
//   - warp 17 (one thread) issues, per query tile, S = Q K^T (M=128, N=128, K=128:
//     8 MMAs) into tensor memory and O += P V (N=128, K=128: 8 MMAs, A = P from tensor
//     memory, B operand MN-major).  The order is fixed, P.V_A(j), S_A(j+1), P.V_B(j),
//     S_B(j+1), so one tile's softmax runs while the tensor core works for the other;
//   - warps 0-15 are the softmax, 8 per query tile: two warps per 32-row quarter, one
//     for keys 0..63 of each key tile and one for keys 64..127.  A thread reads its 64
//     logits from tensor memory and masks them (causal, and past the context); the two
//     halves of a row swap partial maxima through shared memory at a hardware barrier
//     over their 64 threads.  The running max is kept in base-2 units, and O is
//     rescaled in tensor memory only when it grows by more than 8 (2^8: exact up to
//     rounding).  Exponentials are taken two at a time in fp16 (ex2.approx.f16x2: 11
//     significant bits, more than P's 8).  P goes as bf16 over the first 64 columns of
//     S; at the end the halves add up their row sums and store O.
// One CTA per SM: 197 KB of shared memory, all 512 tensor-memory columns (per query
// tile S 128 + O 128).
// Every wait is bounded; on expiry the CTA raises PA_DEV_WAIT_TIMEOUT, drains its own
// copies and MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "pa_internal.h"
#include "pa_ptx.cuh"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

constexpr int kM = 128;            // rows of a query tile
constexpr int kN = 128;            // key tokens per K/V tile
constexpr int kD = 128;            // head dim
constexpr int kQHalf = kM * 128;   // bytes of a 64-column half of a Q tile (16 KB)
constexpr int kKVHalf = kN * 128;  // bytes of a 64-column half of a K or V tile (16 KB)
constexpr int kBox = 16;           // rows per TMA box of K/V (one 16-token run of a block)
constexpr int kNBox = kN / kBox;   // boxes per K/V tile
constexpr int kQT = 2;             // query tiles per CTA, sharing every K/V tile
constexpr int kThreads = 576;      // 8 softmax warps per query tile (two per row), producer, MMA issuer
constexpr int kProdWarp = 16, kMmaWarp = 17;
constexpr uint32_t kTmemCols = 512;  // per query tile: S 0..127 (P over 0..63 once S is read), O 128..255
constexpr uint32_t kLazyRescale = 8; // base-2 units

// Tiles, from a 1024-byte aligned base: Q (two tiles of 32 KB), K and V in two stages
// each (32 KB): 192 KB.  K and V have rings of their own: a K stage is free again as
// soon as the S = Q K^T of both query tiles have run.  The barriers and the exchange
// buffer of the row halves follow the tiles.
constexpr int KST = 2, VST = 2;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + kQT * 2 * kQHalf;
constexpr int OFF_V = OFF_K + KST * 2 * kKVHalf;
constexpr int kTiles = OFF_V + VST * 2 * kKVHalf;
// barriers: q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], per query tile
// {s_full, p_full, o_done}, drain
constexpr int NBAR = 1 + 2 * KST + 2 * VST + kQT * 3 + 1;
constexpr int kXch = 2 * kQT * 2 * 128 * 4;  // partial row maxima (and sums), [tile parity][qt][half][row]
constexpr int kMisc = NBAR * 8 + 16 + kXch;
constexpr int kSmem = (kTiles + 1023 + kMisc + 15) / 16 * 16;
static_assert(kSmem <= 227 * 1024, "one CTA per SM");

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x for two arguments at once: rounded to fp16 on the way in (11 significant bits, as many as the result's)
__device__ __forceinline__ float2 exp2_pair(float x0, float x1)
{
    const __half2 h = __floats2half2_rn(x0, x1);
    uint32_t y;
    asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(*reinterpret_cast<const uint32_t*>(&h)));
    return __half22float2(*reinterpret_cast<const __half2*>(&y));
}

// A barrier over the 64 threads of the two warps that share a row quarter (hardware barrier `id`), returning the
// AND of `v` over them.  Both warps take the same decision from it, so they leave their loop at the same step.
__device__ __forceinline__ bool pair_sync_and(int id, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 64, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// The first 16 of r as 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v)
{
    constexpr int T = kM / G;
    const int pair = (int)gridDim.x - 1 - (int)blockIdx.x;
    const int kvh = blockIdx.y;
    const int s = blockIdx.z;
    const int q0 = __ldg(a.q_start + s);
    const int q1 = __ldg(a.q_start + s + 1);
    const int n = q1 - q0;
    int L = __ldg(a.context_lens + s);
    const int Lcap = a.max_blocks_per_seq * a.block_size;
    if (q0 < 0 || q1 > a.num_query_tokens || n < 0 || n > a.max_query_len || L < n || L > Lcap) {
        if (threadIdx.x == 0 && pair == 0 && kvh == 0) atomicOr(a.status, PA_DEV_BAD_CONTEXT);
        return;
    }
    const int t_lo0 = pair * kQT * T;
    if (t_lo0 >= n) return;
    const int nqt = t_lo0 + T < n ? 2 : 1;
    const int nA = (L - n + min(n, t_lo0 + T) - 1) / kN + 1;
    const int nB = nqt > 1 ? (L - n + min(n, t_lo0 + 2 * T) - 1) / kN + 1 : 0;
    const int ntiles = nqt > 1 ? nB : nA;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTiles);
    uint64_t* q_full = bars;
    uint64_t* k_full = q_full + 1;
    uint64_t* k_empty = k_full + KST;
    uint64_t* v_full = k_empty + KST;
    uint64_t* v_empty = v_full + VST;
    uint64_t* qbars = v_empty + VST;
    uint64_t* drain = qbars + kQT * 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1) + 2;
    float* xch = reinterpret_cast<float*>(drain + 3);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < KST; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < VST; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int qt = 0; qt < kQT; ++qt) {
            mbar_init(&qbars[3 * qt + 0], 1);
            mbar_init(&qbars[3 * qt + 1], 8);
            mbar_init(&qbars[3 * qt + 2], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProdWarp) {
        const uint64_t pol = policy_evict_normal();
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, nqt * 2 * kQHalf);
            for (int qt = 0; qt < nqt; ++qt)
                for (int h = 0; h < 2; ++h)
                    tma_load_3d(smem_u32(smem + OFF_Q + qt * 2 * kQHalf + h * kQHalf), &tmap_q, h * 64, kvh * G,
                                q0 + t_lo0 + qt * T, q_full, pol);
        }
        const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
        auto lookup = [&](int j) -> int {
            const int tok = j * kN + lane * kBox;
            return (j < ntiles && lane < kNBox && tok < L) ? __ldg(table + tok / a.block_size) : 0;
        };
        int next = lookup(0);
        bool ok = true;
        int nk = 0, nv = 0;
        for (int j = 0; j < ntiles && ok; ++j) {
            int phys = next;
            next = lookup(j + 1);
            const int tok0 = j * kN;
            const int nbox = min(kNBox, (L - tok0 + kBox - 1) / kBox);
            const int tok = tok0 + lane * kBox;
            if (lane < nbox && (unsigned)phys >= (unsigned)a.num_blocks) {
                atomicOr(a.status, PA_DEV_BAD_BLOCK);
                phys = 0;
            }
            const int row = (phys * a.num_kv_heads + kvh) * a.block_size + tok % a.block_size;
            const uint32_t tx = (uint32_t)nbox * kBox * 128 * 2;
            const int ks = j % KST;
            if (lane == 0) {
                if (j >= KST && !mbar_wait_bounded(&k_empty[ks], ((j / KST) & 1) ^ 1, abort_flag)) ok = false;
                if (ok) mbar_arrive_expect_tx(&k_full[ks], tx);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            if (lane < nbox)
                for (int h = 0; h < 2; ++h)
                    tma_load_2d(smem_u32(smem + OFF_K + ks * 2 * kKVHalf + h * kKVHalf + lane * kBox * 128), &tmap_k,
                                h * 64, row, &k_full[ks], pol);
            ++nk;
            const int vs = j % VST;
            if (lane == 0) {
                if (j >= VST && !mbar_wait_bounded(&v_empty[vs], ((j / VST) & 1) ^ 1, abort_flag)) ok = false;
                if (ok) mbar_arrive_expect_tx(&v_full[vs], tx);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            if (lane < nbox)
                for (int h = 0; h < 2; ++h)
                    tma_load_2d(smem_u32(smem + OFF_V + vs * 2 * kKVHalf + h * kKVHalf + lane * kBox * 128), &tmap_v,
                                h * 64, row, &v_full[vs], pol);
            ++nv;
        }
        if (lane == 0) {
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            volatile int never = 0;
            if (!mbar_wait_bounded(q_full, 0, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            for (int j = max(0, nk - KST); j < nk; ++j)
                if (!mbar_wait_bounded(&k_full[j % KST], (j / KST) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            for (int j = max(0, nv - VST); j < nv; ++j)
                if (!mbar_wait_bounded(&v_full[j % VST], (j / VST) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else if (warp == kMmaWarp) {
        // MMA issuer, in a fixed order that staggers the two query tiles: P.V_A(j), S_A(j+1),
        // P.V_B(j), S_B(j+1).  Tile A's softmax of tile j+1 then runs while the tensor core
        // does tile B's P.V(j) and S(j+1), and the other way round.
        if (lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(kM, kN, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(kM, kD, true);
            const uint32_t sq = smem_u32(smem + OFF_Q), sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
            auto issue_qk = [&](int qt, int j) {
                const uint32_t qb = sq + qt * 2 * kQHalf;
                const uint32_t kb = sk + (j % KST) * 2 * kKVHalf;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t kk = (k & 3) * 32;
                    umma_bf16_ss(tmem + qt * 256, umma_desc_sw128(qb + (k >> 2) * kQHalf + kk, 16, 1024),
                                 umma_desc_sw128(kb + (k >> 2) * kKVHalf + kk, 16, 1024), idesc_qk, k > 0 ? 1u : 0u);
                }
                umma_commit(&qbars[3 * qt + 0]);
            };
            auto issue_pv = [&](int qt, int j) {
                const uint32_t ts = tmem + qt * 256;
                const uint32_t vb = sv + (j % VST) * 2 * kKVHalf;
#pragma unroll
                for (int k = 0; k < kN / 16; ++k) {
                    umma_bf16_ts(ts + 128, ts + k * 8, umma_desc_sw128(vb + k * 16 * 128, kKVHalf, 1024), idesc_pv,
                                 (j > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&qbars[3 * qt + 2]);
            };
            const int need[kQT] = {nA, nB};
            bool ok = mbar_wait_bounded(q_full, 0, abort_flag) && mbar_wait_bounded(&k_full[0], 0, abort_flag);
            if (ok) {
                tc_fence_after_sync();
                issue_qk(0, 0);
                if (nB > 0) issue_qk(1, 0);
                umma_commit(&k_empty[0]);
            }
            for (int j = 0; j < ntiles && ok; ++j) {
                const bool k_next = j + 1 < ntiles;
                if (!mbar_wait_bounded(&v_full[j % VST], (j / VST) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                for (int qt = 0; qt < kQT && ok; ++qt) {
                    if (j >= need[qt]) continue;
                    if (!mbar_wait_bounded(&qbars[3 * qt + 1], j & 1, abort_flag)) {  // P(j) written
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    issue_pv(qt, j);
                    if (j + 1 < need[qt]) {
                        // S(j+1) goes over the columns P(j) is read from: after P.V(j) has finished
                        if (!mbar_wait_bounded(&k_full[(j + 1) % KST], ((j + 1) / KST) & 1, abort_flag) ||
                            !mbar_wait_bounded(&qbars[3 * qt + 2], j & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        issue_qk(qt, j + 1);
                    }
                }
                if (!ok) break;
                umma_commit(&v_empty[j % VST]);
                if (k_next) umma_commit(&k_empty[(j + 1) % KST]);
            }
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            umma_commit(drain);
            volatile int never = 0;
            if (!mbar_wait_bounded(drain, 0, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else {
        // Softmax: warps 8*qt + 4*half + quarter.  The two warps of a row quarter share its rows, half 0 taking
        // keys 0..63 of each tile and half 1 keys 64..127; they swap partial row maxima through shared memory.
        const int qt = warp >> 3;
        const int half = (warp >> 2) & 1;
        const int r = threadIdx.x & 127;
        const int t256 = threadIdx.x & 255;
        const int t_lo = t_lo0 + qt * T;
        const int ntq = qt == 0 ? nA : nB;
        uint64_t* s_full = &qbars[3 * qt + 0];
        uint64_t* p_full = &qbars[3 * qt + 1];
        uint64_t* o_done = &qbars[3 * qt + 2];
        const int pair_bar = 1 + qt * 4 + (warp & 3);
        const uint32_t tmem_s = tmem + qt * 256;
        const uint32_t tmem_o = tmem_s + 128;
        const int t_local = r / G;
        const int g = r % G;
        const int tq = t_lo + t_local;
        const bool valid_row = t_local < T && tq < n;
        const int lim = valid_row ? (L - n + tq) : -1;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float sl = a.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        constexpr int NC = 2;  // 32-key chunks per half
        auto xslot = [&](int par, int h) -> float* { return xch + ((par * kQT + qt) * 2 + h) * 128 + r; };
        for (int j = 0; j < ntq; ++j) {
            // a failed wait is carried to the pair barrier below, where both warps leave together
            const bool ok_s = ok && mbar_wait_warp(s_full, j & 1, abort_flag);
            tc_fence_after_sync();
            uint32_t sr[NC][32];
#pragma unroll
            for (int c = 0; c < NC; ++c) tmem_ld32(tmem_s + lane_base + half * 64 + c * 32, sr[c]);
            tmem_wait_ld();
            const int kv0 = j * kN + half * 64;
            const float masked = sl >= 0.f ? -INFINITY : INFINITY;
            const bool mask_tile = __any_sync(0xffffffffu, kv0 + 63 > lim);
            if (mask_tile) {
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (kv0 + c * 32 + e > lim) sr[c][e] = __float_as_uint(masked);
            }
            float m0 = masked, m1 = masked, m2 = masked, m3 = masked, m4 = masked, m5 = masked, m6 = masked,
                  m7 = masked;
            if (sl >= 0.f) {
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        m0 = fmaxf(m0, __uint_as_float(sr[c][e + 0]));
                        m1 = fmaxf(m1, __uint_as_float(sr[c][e + 1]));
                        m2 = fmaxf(m2, __uint_as_float(sr[c][e + 2]));
                        m3 = fmaxf(m3, __uint_as_float(sr[c][e + 3]));
                        m4 = fmaxf(m4, __uint_as_float(sr[c][e + 4]));
                        m5 = fmaxf(m5, __uint_as_float(sr[c][e + 5]));
                        m6 = fmaxf(m6, __uint_as_float(sr[c][e + 6]));
                        m7 = fmaxf(m7, __uint_as_float(sr[c][e + 7]));
                    }
                m0 = fmaxf(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)), fmaxf(fmaxf(m4, m5), fmaxf(m6, m7)));
            } else {
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        m0 = fminf(m0, __uint_as_float(sr[c][e + 0]));
                        m1 = fminf(m1, __uint_as_float(sr[c][e + 1]));
                        m2 = fminf(m2, __uint_as_float(sr[c][e + 2]));
                        m3 = fminf(m3, __uint_as_float(sr[c][e + 3]));
                        m4 = fminf(m4, __uint_as_float(sr[c][e + 4]));
                        m5 = fminf(m5, __uint_as_float(sr[c][e + 5]));
                        m6 = fminf(m6, __uint_as_float(sr[c][e + 6]));
                        m7 = fminf(m7, __uint_as_float(sr[c][e + 7]));
                    }
                m0 = fminf(fminf(fminf(m0, m1), fminf(m2, m3)), fminf(fminf(m4, m5), fminf(m6, m7)));
            }
            // swap the partial maxima; the barrier also orders this half's S reads before the other half's P
            // stores over S's first 64 columns
            *xslot(j & 1, half) = m0;
            tc_fence_before_sync();
            if (!pair_sync_and(pair_bar, ok_s)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            const float other = *xslot(j & 1, half ^ 1);
            const float mraw = sl >= 0.f ? fmaxf(m0, other) : fminf(m0, other);
            const float mx = mraw == masked ? -INFINITY : mraw * sl;
            const float m_new = fmaxf(m_used, mx);
            const bool rescale = m_used != -INFINITY && m_new > m_used + (float)kLazyRescale;
            const bool rescale_warp = __any_sync(0xffffffffu, rescale) != 0;
            const float alpha = rescale ? fast_exp2(m_used - m_new) : 1.f;
            if (rescale || m_used == -INFINITY) m_used = m_new;
            const float mref = m_used == -INFINITY ? 0.f : m_used;
            float rs0 = 0.f, rs1 = 0.f, rs2 = 0.f, rs3 = 0.f;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
#pragma unroll
                for (int e2 = 0; e2 < 16; ++e2) {
                    const float2 pp = exp2_pair(fmaf(__uint_as_float(sr[c][2 * e2]), sl, -mref),
                                                fmaf(__uint_as_float(sr[c][2 * e2 + 1]), sl, -mref));
                    float p0 = pp.x, p1 = pp.y;
                    if (mask_tile) {
                        const int kv = kv0 + c * 32 + 2 * e2;
                        p0 = kv <= lim ? p0 : 0.f;
                        p1 = kv + 1 <= lim ? p1 : 0.f;
                    }
                    if (e2 & 1) {
                        rs2 += p0;
                        rs3 += p1;
                    } else {
                        rs0 += p0;
                        rs1 += p1;
                    }
                    sr[c][e2] = pack_bf16(p0, p1);
                }
                tmem_st16(tmem_s + lane_base + half * 32 + c * 16, sr[c]);
            }
            if (rescale_warp) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem_o + lane_base + half * 64 + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tmem_o + lane_base + half * 64 + c * 32, o);
                }
            }
            tmem_wait_st();
            l = l * alpha + ((rs0 + rs1) + (rs2 + rs3));
            if (j * kN + kN > L) {
                // V rows past the context: their P is 0, and 0 must not meet a NaN left in the pool
                const bool v_ok = mbar_wait_warp(&v_full[j % VST], (j / VST) & 1, abort_flag);
                if (!v_ok) ok = false;
                const int first = max(0, L - j * kN);
                const int chunks = v_ok ? (kN - first) * 16 : 0;
                for (int i = t256; i < chunks; i += 256) {
                    const int row = first + (i >> 4);
                    const int h = (i >> 3) & 1;
                    *reinterpret_cast<uint4*>(smem + OFF_V + (j % VST) * 2 * kKVHalf + h * kKVHalf + row * 128 +
                                              (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (ntq > 0) {
            // the row sum is split between the halves as well; both warps of the pair always get here
            *xslot(ntq & 1, half) = l;
            if (!pair_sync_and(pair_bar, ok)) ok = false;
            if (ok) l += *xslot(ntq & 1, half ^ 1);
        }
        if (ntq == 0) {
        } else if (ok && mbar_wait_warp(o_done, (ntq - 1) & 1, abort_flag)) {
            tc_fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                                 ((size_t)(q0 + tq) * a.num_heads + (size_t)kvh * G + g) * kD + half * 64;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem_o + lane_base + half * 64 + c * 32, o);
                tmem_wait_ld();
                if (valid_row) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 pk;
                        pk.x = pack_bf16(__uint_as_float(o[v4 * 8 + 0]) * inv, __uint_as_float(o[v4 * 8 + 1]) * inv);
                        pk.y = pack_bf16(__uint_as_float(o[v4 * 8 + 2]) * inv, __uint_as_float(o[v4 * 8 + 3]) * inv);
                        pk.z = pack_bf16(__uint_as_float(o[v4 * 8 + 4]) * inv, __uint_as_float(o[v4 * 8 + 5]) * inv);
                        pk.w = pack_bf16(__uint_as_float(o[v4 * 8 + 6]) * inv, __uint_as_float(o[v4 * 8 + 7]) * inv);
                        *reinterpret_cast<uint4*>(out + c * 32 + v4 * 8) = pk;
                    }
                }
            }
        } else {
            ok = false;
        }
        if (!ok) {
            if (lane == 0) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// q [Nq][Hq][D] as a 3-D bf16 tensor (D, Hq, Nq); boxes of 64 columns x G heads x
// 128/G tokens, 128-byte swizzle: one box fills a 64-column half of the Q tile with
// rows ordered (token, head).
cudaError_t q_tensor_map(CUtensorMap* out, const void* q, int num_tokens, int num_heads, int G)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    std::memset(out, 0, sizeof(*out));
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)num_heads, (cuuint64_t)num_tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)num_heads * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(kM / G)};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int G>
cudaError_t launch_g(const PrefillArgs& a, int num_query_tokens, int max_query_len, cudaStream_t stream)
{
    CUtensorMap tq, tk, tv;
    cudaError_t e = q_tensor_map(&tq, a.q, num_query_tokens, a.num_heads, G);
    if (e != cudaSuccess) return e;
    const uint64_t rows = (uint64_t)a.num_blocks * a.num_kv_heads * a.block_size;
    if ((e = tensor_map(&tk, a.k_cache, rows, kD, kBox)) != cudaSuccess) return e;
    if ((e = tensor_map(&tv, a.v_cache, rows, kD, kBox)) != cudaSuccess) return e;
    // the kernel's attributes, set once per device (setting them twice is harmless, so
    // two threads racing to the first call need no lock)
    static std::atomic<bool> attr_done[64] = {};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (!attr_done[dev & 63].load()) {
        e = cudaFuncSetAttribute(prefill_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(prefill_tc_kernel<G>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        attr_done[dev & 63].store(true);
    }
    constexpr int T = kM / G;
    const dim3 grid((unsigned)((max_query_len + kQT * T - 1) / (kQT * T)), (unsigned)a.num_kv_heads,
                    (unsigned)a.num_seqs);
    prefill_tc_kernel<G><<<grid, kThreads, kSmem, stream>>>(a, tq, tk, tv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, int group, int num_query_tokens, int max_query_len,
                           cudaStream_t stream)
{
    if (a.num_seqs == 0 || max_query_len == 0 || num_query_tokens == 0) return cudaSuccess;
    switch (group) {
        case 1: return launch_g<1>(a, num_query_tokens, max_query_len, stream);
        case 2: return launch_g<2>(a, num_query_tokens, max_query_len, stream);
        case 4: return launch_g<4>(a, num_query_tokens, max_query_len, stream);
        case 8: return launch_g<8>(a, num_query_tokens, max_query_len, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pa
