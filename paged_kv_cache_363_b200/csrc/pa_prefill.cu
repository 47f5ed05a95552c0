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
// A CTA owns one (sequence, kv head, query tile).  The tile's 128 rows are T query
// tokens x G query heads of the kv head's group (T = 128 / G), so every K/V byte the
// CTA loads serves all G heads.  It walks the keys in tiles of 64 tokens:
//   - warp 4 stages Q once and each K and V tile by TMA, one 16-row box per (16-token
//     run of a physical block, 64 columns), 128-byte swizzle, K in three stages and V
//     in two; lane i looks up and issues box i of the tile;
//   - warp 5 (one thread) issues S = Q K^T (M=128, N=64, K=128: 8 MMAs) into tensor
//     memory, and O += P V (N=128, K=64: 4 MMAs, A = P from tensor memory, B operand
//     MN-major) once P is ready; the next
//     tile's S is issued as soon as the softmax has read this one, so it overlaps the
//     softmax;
//   - warps 0-3 (a thread per row) read S from tensor memory, mask (causal and past
//     the context), keep the running max in base-2 units, rescale O in tensor memory
//     only when the max grows by more than 8 (2^8: exact up to rounding, fewer
//     rescales), write P as bf16 into tensor memory (two buffers, so the next tile's
//     P is written while this tile's P.V runs), and at the end normalise O and store it.
// Two CTAs share an SM (113 KB of shared memory and 256 tensor-memory columns each),
// so one CTA's softmax overlaps the other's matrix multiplies.
// Every wait is bounded; on expiry the CTA raises PA_DEV_WAIT_TIMEOUT, drains its own
// copies and MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "pa_internal.h"
#include "pa_ptx.cuh"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

constexpr int kM = 128;            // tile rows
constexpr int kN = 64;             // key tokens per tile
constexpr int kD = 128;            // head dim
constexpr int kQHalf = kM * 128;   // bytes of a 64-column half of the Q tile (16 KB)
constexpr int kKVHalf = kN * 128;  // bytes of a 64-column half of a K or V tile (8 KB)
constexpr int kBox = 16;           // rows per TMA box of K/V (one 16-token run of a block)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;  // S: 0..63, P: 64..95 and 96..127, O: 128..255 (two CTAs fill the 512)
constexpr uint32_t kLazyRescale = 8; // base-2 units

// Tiles, from a 1024-byte aligned base: Q (32 KB), K in three stages and V in two
// (16 KB each): 112 KB.  K and V have rings of their own: a K stage is free again as
// soon as its S = Q K^T has run, so the next K tiles load a whole softmax earlier than
// a shared K/V stage (freed only by P.V) would allow.  P lives in tensor memory (two
// buffers, the A operand of P.V).  The barriers go in the alignment slack when it has
// room, else after the tiles, so the request fits two CTAs per SM
// (2 x (113 KB + 1 KB reserved) = 228 KB).
constexpr int KST = 3, VST = 2;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + 2 * kQHalf;
constexpr int OFF_V = OFF_K + KST * 2 * kKVHalf;
constexpr int kTiles = OFF_V + VST * 2 * kKVHalf;
// barriers: q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full, s_free, p_full, o_done[2], drain
constexpr int NBAR = 1 + 2 * KST + 2 * VST + 6;
constexpr int kMisc = 160;          // barriers, TMEM base, abort flag
constexpr int kSmem = 113 * 1024;
static_assert(kTiles + 1023 <= kSmem, "tiles fit with any base alignment");
static_assert((kMisc - 1) + kTiles + kMisc <= kSmem, "misc after the tiles when the slack is short");
static_assert(NBAR * 8 + 16 <= kMisc, "misc area");

// 2^x by the hardware approximation (ex2.approx, relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <int G>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v)
{
    constexpr int T = kM / G;  // query tokens per tile
    const int tile = (int)gridDim.x - 1 - (int)blockIdx.x;  // the tiles with the most keys start first
    const int kvh = blockIdx.y;
    const int s = blockIdx.z;
    const int q0 = __ldg(a.q_start + s);
    const int q1 = __ldg(a.q_start + s + 1);
    const int n = q1 - q0;
    int L = __ldg(a.context_lens + s);
    const int Lcap = a.max_blocks_per_seq * a.block_size;
    // device data checked before anything is read through it or stored: the
    // sequence's query rows must lie inside q and out, in order, and within the
    // launch's rows per sequence; its context must hold them and fit its table row.
    // A bad sequence is flagged and skipped whole: its output rows stay untouched.
    if (q0 < 0 || q1 > a.num_query_tokens || n < 0 || n > a.max_query_len || L < n || L > Lcap) {
        if (threadIdx.x == 0 && tile == 0 && kvh == 0) atomicOr(a.status, PA_DEV_BAD_CONTEXT);
        return;
    }
    const int t_lo = tile * T;
    if (t_lo >= n) return;  // whole CTA, before any shared state exists
    const int t_hi = min(n, t_lo + T);
    const int p_max = L - n + t_hi - 1;  // last query position of the tile
    const int ntiles = p_max / kN + 1;

    extern __shared__ unsigned char smem_raw[];
    const uint32_t slack = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    unsigned char* smem = smem_raw + slack;
    unsigned char* misc = slack >= (uint32_t)kMisc ? smem_raw : smem + kTiles;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = q_full + 1;        // [KST]
    uint64_t* k_empty = k_full + KST;     // [KST]
    uint64_t* v_full = k_empty + KST;     // [VST]
    uint64_t* v_empty = v_full + VST;     // [VST]
    uint64_t* s_full = v_empty + VST;
    uint64_t* s_free = s_full + 1;
    uint64_t* p_full = s_free + 1;
    uint64_t* o_done = p_full + 1;        // [2]: P.V of the tiles using P buffer 0 / 1
    uint64_t* drain = o_done + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + NBAR * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + NBAR * 8 + 8);
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
        mbar_init(s_full, 1);
        mbar_init(s_free, 4);
        mbar_init(p_full, 4);
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_s = tmem;
    const uint32_t tmem_p = tmem + 64;  // + 32 * buffer
    const uint32_t tmem_o = tmem + 128;

    if (warp == 4) {
        // ---------------- producer: Q once, then K/V tiles.  Lane i looks up the
        // physical block of the tile's i-th 16-token box and issues its copies, so
        // the table reads of a tile overlap instead of queueing behind each other.
        const uint64_t pol = policy_evict_normal();
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, 2 * kQHalf);
            for (int h = 0; h < 2; ++h)
                tma_load_3d(smem_u32(smem + OFF_Q + h * kQHalf), &tmap_q, h * 64, kvh * G, q0 + t_lo, q_full, pol);
        }
        const int32_t* table = a.block_tables + (size_t)s * a.max_blocks_per_seq;
        bool ok = true;
        for (int j = 0; j < ntiles && ok; ++j) {
            const int tok0 = j * kN;
            const int nbox = min(kN / kBox, (L - tok0 + kBox - 1) / kBox);
            const int tok = tok0 + lane * kBox;
            int phys = 0;
            if (lane < nbox) {
                phys = __ldg(table + tok / a.block_size);
                if ((unsigned)phys >= (unsigned)a.num_blocks) {
                    atomicOr(a.status, PA_DEV_BAD_BLOCK);
                    phys = 0;
                }
            }
            const int row = (phys * a.num_kv_heads + kvh) * a.block_size + tok % a.block_size;
            const uint32_t tx = (uint32_t)nbox * kBox * 128 * 2;  // both halves of the boxes
            // K tile j into K stage j % KST, free once S of tile j - KST has run
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
            // V tile j into V stage j % VST, free once P.V of tile j - VST has run
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
        }
        if (lane == 0) {
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // no copy may still be landing in shared memory at exit
            volatile int never = 0;
            if (!mbar_wait_bounded(q_full, 0, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            for (int j = max(0, ntiles - KST); j < ntiles; ++j)
                if (!mbar_wait_bounded(&k_full[j % KST], (j / KST) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            for (int j = max(0, ntiles - VST); j < ntiles; ++j)
                if (!mbar_wait_bounded(&v_full[j % VST], (j / VST) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else if (warp == 5) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(kM, kN, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(kM, kD, true);
            const uint32_t sq = smem_u32(smem + OFF_Q), sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
            bool ok = mbar_wait_bounded(q_full, 0, abort_flag) && mbar_wait_bounded(&k_full[0], 0, abort_flag);
            auto issue_qk = [&](int j) {
                const uint32_t kb = sk + (j % KST) * 2 * kKVHalf;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t kk = (k & 3) * 32;
                    umma_bf16_ss(tmem_s, umma_desc_sw128(sq + (k >> 2) * kQHalf + kk, 16, 1024),
                                 umma_desc_sw128(kb + (k >> 2) * kKVHalf + kk, 16, 1024), idesc_qk, k > 0 ? 1u : 0u);
                }
                umma_commit(s_full);
                umma_commit(&k_empty[j % KST]);
            };
            if (ok) {
                tc_fence_after_sync();
                issue_qk(0);
            }
            for (int j = 0; j < ntiles && ok; ++j) {
                if (j + 1 < ntiles) {
                    if (!mbar_wait_bounded(&k_full[(j + 1) % KST], ((j + 1) / KST) & 1, abort_flag) ||
                        !mbar_wait_bounded(s_free, j & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    issue_qk(j + 1);
                }
                if (!mbar_wait_bounded(p_full, j & 1, abort_flag) ||
                    !mbar_wait_bounded(&v_full[j % VST], (j / VST) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t vb = sv + (j % VST) * 2 * kKVHalf;
#pragma unroll
                for (int k = 0; k < kN / 16; ++k) {
                    umma_bf16_ts(tmem_o, tmem_p + (j & 1) * 32 + k * 8,
                                 umma_desc_sw128(vb + k * 16 * 128, kKVHalf, 1024), idesc_pv,
                                 (j > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&o_done[j & 1]);
                umma_commit(&v_empty[j % VST]);
            }
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // every MMA issued here has completed before tensor memory is freed
            umma_commit(drain);
            volatile int never = 0;
            if (!mbar_wait_bounded(drain, 0, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else {
        // ---------------- softmax warps: thread r owns tile row r (TMEM lane r)
        const int r = threadIdx.x;
        const int t_local = r / G;
        const int g = r % G;
        const int tq = t_lo + t_local;
        const bool valid_row = t_local < T && tq < n;
        const int lim = valid_row ? (L - n + tq) : -1;  // last key this row may see
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float sl = a.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            if (!mbar_wait_warp(s_full, j & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            constexpr int NC = kN / 32;  // 32-column chunks of the S row
            uint32_t sr[NC][32];
#pragma unroll
            for (int c = 0; c < NC; ++c) tmem_ld32(tmem_s + lane_base + c * 32, sr[c]);
            tmem_wait_ld();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free);
            const int kv0 = j * kN;
            // Work on the raw logits: the scale and the max subtraction fold into one FMA
            // below.  Keys past a row's limit become the value that scales to -inf; only
            // tiles that cross some row's limit in this warp pay for the mask.
            const float masked = sl >= 0.f ? -INFINITY : INFINITY;
            const bool mask_tile = __any_sync(0xffffffffu, kv0 + kN - 1 > lim);
            if (mask_tile) {
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (kv0 + c * 32 + e > lim) sr[c][e] = __float_as_uint(masked);
            }
            // eight independent partial maxima (short dependency chains), then a tree
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
            const float mraw = m0;
            const float mx = mraw == masked ? -INFINITY : mraw * sl;  // the row's max in base-2 units
            const float m_new = fmaxf(m_used, mx);
            const bool rescale = m_used != -INFINITY && m_new > m_used + (float)kLazyRescale;
            // the whole warp takes the O round trip when any of its rows needs it
            const bool rescale_warp = __any_sync(0xffffffffu, rescale) != 0;
            // P buffer j & 1 is free once the P.V of tile j - 2 has finished; O is stable
            // for a rescale once the P.V of tile j - 1 has (each buffer has its own
            // barrier, whose next phase is never more than one ahead of the wait)
            if (j >= 2 && !mbar_wait_warp(&o_done[j & 1], ((j - 2) >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            if (rescale_warp && j >= 1 && !mbar_wait_warp(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            if (rescale_warp) {
                const float alpha = rescale ? fast_exp2(m_used - m_new) : 1.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem_o + lane_base + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tmem_o + lane_base + c * 32, o);
                }
                tmem_wait_st();
                l *= alpha;
            }
            if (rescale || m_used == -INFINITY) m_used = m_new;
            const float mref = m_used == -INFINITY ? 0.f : m_used;  // a row with no key yet: every x is -inf
            // P = 2^(raw * scale - m) as bf16 pairs into this lane of P buffer j & 1 (32 columns);
            // the row sum takes P before rounding (two partial sums for more parallel adds)
            float rs0 = 0.f, rs1 = 0.f, rs2 = 0.f, rs3 = 0.f;  // independent partial sums
            uint32_t w[32];
            if (!mask_tile) {
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        const float p0 = fast_exp2(fmaf(__uint_as_float(sr[c][2 * e2]), sl, -mref));
                        const float p1 = fast_exp2(fmaf(__uint_as_float(sr[c][2 * e2 + 1]), sl, -mref));
                        if (e2 & 1) {
                            rs2 += p0;
                            rs3 += p1;
                        } else {
                            rs0 += p0;
                            rs1 += p1;
                        }
                        w[c * 16 + e2] = pack_bf16(p0, p1);
                    }
            } else {
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        const int kv = kv0 + c * 32 + 2 * e2;
                        const float p0 = kv <= lim ? fast_exp2(fmaf(__uint_as_float(sr[c][2 * e2]), sl, -mref)) : 0.f;
                        const float p1 =
                            kv + 1 <= lim ? fast_exp2(fmaf(__uint_as_float(sr[c][2 * e2 + 1]), sl, -mref)) : 0.f;
                        if (e2 & 1) {
                            rs2 += p0;
                            rs3 += p1;
                        } else {
                            rs0 += p0;
                            rs1 += p1;
                        }
                        w[c * 16 + e2] = pack_bf16(p0, p1);
                    }
            }
            const float rowsum = (rs0 + rs1) + (rs2 + rs3);
            tmem_st32(tmem_p + (j & 1) * 32 + lane_base, w);
            tmem_wait_st();
            l += rowsum;
            // keys past the context in this tile: zero their V rows (0-weights must meet finite values)
            if (kv0 + kN > L) {
                // the tile's V copies (boxes with tokens past the context included) have landed
                if (!mbar_wait_warp(&v_full[j % VST], (j / VST) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                unsigned char* vb = smem + OFF_V + (j % VST) * 2 * kKVHalf;
                const int first = max(0, L - kv0);
                const int chunks = (kN - first) * 16;  // 16-byte chunks over both halves
                for (int i = r; i < chunks; i += 128) {
                    const int row = first + (i >> 4);
                    const int h = (i >> 3) & 1;
                    *reinterpret_cast<uint4*>(vb + h * kKVHalf + row * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (ok && mbar_wait_warp(&o_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, abort_flag)) {
            tc_fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                                 ((size_t)(q0 + tq) * a.num_heads + (size_t)kvh * G + g) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem_o + lane_base + c * 32, o);
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
    if (warp == 5) tmem_dealloc(tmem, kTmemCols);
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
    const dim3 grid((unsigned)((max_query_len + T - 1) / T), (unsigned)a.num_kv_heads, (unsigned)a.num_seqs);
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
