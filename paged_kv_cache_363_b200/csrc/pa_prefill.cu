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
// A work item is one (sequence, kv head) and two query tiles A and B of 128 rows each.
// A tile's rows are T query tokens x G query heads of the kv head's group (T = 128 / G),
// so every K/V byte loaded serves both tiles and all G heads.  With a workspace
// (pa_prefill_ws) one CTA per SM claims items from a counter, and starts an item's Q
// load and first S while its previous item ends; without one (pa_prefill) CTA b runs
// item b alone.  Items go in chunks of 16 (sequence, kv head) groups, the last query
// tokens of the chunk's groups first, so the CTAs that run together share a few
// groups' K/V in L2.  An item walks the keys in tiles of 128 tokens:
//   - warp 16 claims the items and passes them, with their geometry, through a ring of
//     two shared-memory slots; it stages both Q tiles once per item and each K and V
//     tile by TMA, one 16-row box per (16-token run of a physical block, 64 columns),
//     128-byte swizzle, K and V in two 32 KB stages each (the rings run on across
//     items); lane i looks up and issues box i of the tile;
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
//     rounding).  The exponent arguments are formed two at a time (fma.rn.f32x2), the
//     exponentials in fp32 (an fp16 pair costs the transcendental unit as much as two
//     fp32 ones and needs conversions both ways).  P goes as bf16 over the first 64
//     columns of S; at the end the halves add up their row sums and store O.
// One CTA per SM: 197 KB of shared memory, all 512 tensor-memory columns (per query
// tile S 128 + O 128).  A tile's O is taken by its next item only after the softmax has
// read it out, and its S only after the previous P.V.
// Every wait is bounded; on expiry the CTA raises PA_DEV_WAIT_TIMEOUT, drains its own
// copies and MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
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
constexpr int kQT = 2;             // query tiles per work item, sharing every K/V tile
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
constexpr int IR = 2;  // item ring: the item in work and the next
constexpr int kChunkGroups = 16;  // (sequence, kv head) groups whose items are interleaved
// barriers: q_full, q_empty, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], per query tile
// {s_full, p_full, o_done, o_free}, drain, it_full[IR], it_empty[IR]
constexpr int NBAR = 2 + 2 * KST + 2 * VST + kQT * 4 + 1 + 2 * IR;
constexpr int kXch = 2 * kQT * 2 * 128 * 4;  // partial row maxima (and sums), [tile parity][qt][half][row]
// after the barriers: TMEM address and abort flag (16 bytes), the item slots, the exchange buffer
constexpr int kSlotInts = 16;
constexpr int kMisc = NBAR * 8 + 16 + 4 * IR * kSlotInts + kXch;
constexpr int kSmem = (kTiles + 1023 + kMisc + 15) / 16 * 16;
static_assert(kSmem <= 227 * 1024, "one CTA per SM");

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// a pair of floats in one 64-bit register, for the f32x2 instructions
__device__ __forceinline__ uint64_t pack2f(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

// (x0, x1) = (s0, s1) * b + c, elementwise over the pairs b and c, in one instruction
__device__ __forceinline__ void ffma2(float& x0, float& x1, uint32_t s0, uint32_t s1, uint64_t b, uint64_t c)
{
    asm("{\n\t.reg .b64 ra, rd;\n\tmov.b64 ra, {%2, %3};\n\t"
        "fma.rn.f32x2 rd, ra, %4, %5;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(x0), "=f"(x1)
        : "r"(s0), "r"(s1), "l"(b), "l"(c));
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

// One work item: query tokens [t_lo0, t_lo0 + 2T) of sequence s (two query tiles of T tokens x G heads) for
// kv head kvh.  Items are numbered by chunks of kChunkGroups (sequence, kv head) groups, and inside a chunk
// with the last query tokens (which see the most keys) first.  With a counter (a.sched) a grid of one CTA per
// SM claims them in that order, so a CTA that finishes early takes more; without one, CTA b takes item b
// alone.  The producer warp claims the items and hands them to the MMA thread and the softmax warps through
// a ring of IR slots in shared memory.
struct Item {
    int s, kvh, pair, q0, n, L, t_lo0, nqt, nA, nB, ntiles;
    bool bad;
};

// An item's geometry in its ring slot (after the item and ring-position words), written by the producer so
// that the MMA thread and the softmax warps read it from shared memory instead of global memory.
__device__ __forceinline__ void put_item(int* p, const Item& it)
{
    p[2] = it.s; p[3] = it.kvh; p[4] = it.pair; p[5] = it.q0; p[6] = it.n; p[7] = it.L; p[8] = it.t_lo0;
    p[9] = it.nqt; p[10] = it.nA; p[11] = it.nB; p[12] = it.ntiles;
}
__device__ __forceinline__ void get_item(const volatile int* p, Item& it)
{
    it.s = p[2]; it.kvh = p[3]; it.pair = p[4]; it.q0 = p[5]; it.n = p[6]; it.L = p[7]; it.t_lo0 = p[8];
    it.nqt = p[9]; it.nA = p[10]; it.nB = p[11]; it.ntiles = p[12]; it.bad = false;
}

template <int G>
__device__ __forceinline__ bool item_geom(const PrefillArgs& a, int npairs, int item, Item& it)
{
    constexpr int T = kM / G;
    // groups = (sequence, kv head) pairs, kChunkGroups at a time; inside a chunk the last query tokens come first,
    // across its groups.  The CTAs that run together then share a few groups' K/V, which stays in L2.
    const int ngroups = a.num_seqs * a.num_kv_heads;
    const int chunk = item / (kChunkGroups * npairs);
    const int cg = min(kChunkGroups, ngroups - chunk * kChunkGroups);  // groups in this chunk
    const int idx = item - chunk * kChunkGroups * npairs;
    it.pair = npairs - 1 - idx / cg;
    const int grp = chunk * kChunkGroups + idx % cg;
    it.s = grp / a.num_kv_heads;
    it.kvh = grp % a.num_kv_heads;
    it.q0 = __ldg(a.q_start + it.s);
    const int q1 = __ldg(a.q_start + it.s + 1);
    it.n = q1 - it.q0;
    it.L = __ldg(a.context_lens + it.s);
    const int Lcap = a.max_blocks_per_seq * a.block_size;
    it.bad = it.q0 < 0 || q1 > a.num_query_tokens || it.n < 0 || it.n > a.max_query_len || it.L < it.n ||
             it.L > Lcap;
    it.t_lo0 = it.pair * kQT * T;
    if (it.bad || it.t_lo0 >= it.n) return false;
    it.nqt = it.t_lo0 + T < it.n ? 2 : 1;
    it.nA = (it.L - it.n + min(it.n, it.t_lo0 + T) - 1) / kN + 1;
    it.nB = it.nqt > 1 ? (it.L - it.n + min(it.n, it.t_lo0 + 2 * T) - 1) / kN + 1 : 0;
    it.ntiles = it.nqt > 1 ? it.nB : it.nA;
    return true;
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                      int npairs)
{
    constexpr int T = kM / G;
    const int nitems = npairs * a.num_seqs * a.num_kv_heads;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTiles);
    uint64_t* q_full = bars;
    uint64_t* q_empty = q_full + 1;
    uint64_t* k_full = q_empty + 1;
    uint64_t* k_empty = k_full + KST;
    uint64_t* v_full = k_empty + KST;
    uint64_t* v_empty = v_full + VST;
    uint64_t* qbars = v_empty + VST;
    uint64_t* drain = qbars + kQT * 4;
    uint64_t* it_full = drain + 1;    // item slot written (producer)
    uint64_t* it_empty = it_full + IR;  // item slot read (MMA thread and the 16 softmax warps)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(it_empty + IR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(it_empty + IR) + 2;
    // [IR][kSlotInts]: the item (-1: the end), the ring position of its first K/V tile, its geometry
    int* item_slot = reinterpret_cast<int*>(it_empty + IR) + 4;
    float* xch = reinterpret_cast<float*>(item_slot + IR * kSlotInts);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < KST; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < VST; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int qt = 0; qt < kQT; ++qt) {
            mbar_init(&qbars[4 * qt + 0], 1);  // s_full: S = Q.K^T in tensor memory
            mbar_init(&qbars[4 * qt + 1], 8);  // p_full: P written by the tile's 8 softmax warps
            mbar_init(&qbars[4 * qt + 2], 1);  // o_done: P.V finished
            mbar_init(&qbars[4 * qt + 3], 8);  // o_free: the item's output read out of tensor memory
        }
        mbar_init(drain, 1);
        for (int i = 0; i < IR; ++i) {
            mbar_init(&it_full[i], 1);
            mbar_init(&it_empty[i], 1 + 16);
        }
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
        bool ok = true;
        int gt = 0;          // K/V tiles of this CTA's items so far: the rings' position
        int nk = 0, nv = 0;  // K and V tile copies issued (they differ only after a failed wait)
        int nit = 0;         // items whose Q was loaded
        int claimed = 0;     // claims made (static grid: one)
        for (;;) {
            // claim the next item with work (lane 0), skipping empty items and flagging bad sequences
            int item = nitems;
            Item it;
            if (lane == 0) {
                for (;;) {
                    item = a.sched ? (int)atomicAdd(a.sched, 1u) : (claimed == 0 ? (int)blockIdx.x : nitems);
                    ++claimed;
                    if (item >= nitems) break;
                    if (item_geom<G>(a, npairs, item, it)) break;
                    if (it.bad && it.pair == 0 && it.kvh == 0) atomicOr(a.status, PA_DEV_BAD_CONTEXT);
                }
                // hand it out (or the end, as -1) once every reader is done with the slot's last item
                if (nit >= IR && !mbar_wait_bounded(&it_empty[nit % IR], ((nit / IR) & 1) ^ 1, abort_flag))
                    ok = false;
                if (ok) {
                    int* sp = item_slot + (nit % IR) * kSlotInts;
                    sp[0] = item < nitems ? item : -1;
                    sp[1] = gt;
                    if (item < nitems) put_item(sp, it);
                    mbar_arrive(&it_full[nit % IR]);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            item = __shfl_sync(0xffffffffu, item, 0);
            if (!ok || item >= nitems) break;
            __syncwarp();  // lane 0's slot writes are visible to the warp
            get_item(item_slot + (nit % IR) * kSlotInts, it);
            // Q of this item goes over the last one's once every Q.K^T that read it has finished
            if (lane == 0) {
                if (nit > 0 && !mbar_wait_bounded(q_empty, (nit - 1) & 1, abort_flag)) ok = false;
                if (ok) {
                    mbar_arrive_expect_tx(q_full, it.nqt * 2 * kQHalf);
                    for (int qt = 0; qt < it.nqt; ++qt)
                        for (int h = 0; h < 2; ++h)
                            tma_load_3d(smem_u32(smem + OFF_Q + qt * 2 * kQHalf + h * kQHalf), &tmap_q, h * 64,
                                        it.kvh * G, it.q0 + it.t_lo0 + qt * T, q_full, pol);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            ++nit;
            const int32_t* table = a.block_tables + (size_t)it.s * a.max_blocks_per_seq;
            auto lookup = [&](int j) -> int {
                const int tok = j * kN + lane * kBox;
                return (j < it.ntiles && lane < kNBox && tok < it.L) ? __ldg(table + tok / a.block_size) : 0;
            };
            int next = lookup(0);
            for (int j = 0; j < it.ntiles; ++j) {
                int phys = next;
                next = lookup(j + 1);
                const int g = gt + j;
                const int tok0 = j * kN;
                const int nbox = min(kNBox, (it.L - tok0 + kBox - 1) / kBox);
                const int tok = tok0 + lane * kBox;
                if (lane < nbox && (unsigned)phys >= (unsigned)a.num_blocks) {
                    atomicOr(a.status, PA_DEV_BAD_BLOCK);
                    phys = 0;
                }
                const int row = (phys * a.num_kv_heads + it.kvh) * a.block_size + tok % a.block_size;
                const uint32_t tx = (uint32_t)nbox * kBox * 128 * 2;
                const int ks = g % KST;
                if (lane == 0) {
                    if (g >= KST && !mbar_wait_bounded(&k_empty[ks], ((g / KST) & 1) ^ 1, abort_flag)) ok = false;
                    if (ok) mbar_arrive_expect_tx(&k_full[ks], tx);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (lane < nbox)
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d(smem_u32(smem + OFF_K + ks * 2 * kKVHalf + h * kKVHalf + lane * kBox * 128),
                                    &tmap_k, h * 64, row, &k_full[ks], pol);
                ++nk;
                const int vs = g % VST;
                if (lane == 0) {
                    if (g >= VST && !mbar_wait_bounded(&v_empty[vs], ((g / VST) & 1) ^ 1, abort_flag)) ok = false;
                    if (ok) mbar_arrive_expect_tx(&v_full[vs], tx);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (lane < nbox)
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d(smem_u32(smem + OFF_V + vs * 2 * kKVHalf + h * kKVHalf + lane * kBox * 128),
                                    &tmap_v, h * 64, row, &v_full[vs], pol);
                ++nv;
            }
            gt += it.ntiles;
        }
        if (lane == 0) {
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // nothing may still be landing in shared memory when the CTA exits
            volatile int never = 0;
            if (nit > 0 && !mbar_wait_bounded(q_full, (nit - 1) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            // a copy older than the last ring's worth had its stage released, so it has landed
            for (int g = max(0, nk - KST); g < nk; ++g)
                if (!mbar_wait_bounded(&k_full[g % KST], (g / KST) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            for (int g = max(0, nv - VST); g < nv; ++g)
                if (!mbar_wait_bounded(&v_full[g % VST], (g / VST) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else if (warp == kMmaWarp) {
        // MMA issuer, in a fixed order that staggers the two query tiles: P.V_A(j), S_A(j+1),
        // P.V_B(j), S_B(j+1).  Tile A's softmax of tile j+1 then runs while the tensor core
        // does tile B's P.V(j) and S(j+1), and the other way round.
        if (lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(kM, kN, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(kM, kD, true);
            const uint32_t sq = smem_u32(smem + OFF_Q), sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
            auto issue_qk = [&](int qt, int g) {
                const uint32_t qb = sq + qt * 2 * kQHalf;
                const uint32_t kb = sk + (g % KST) * 2 * kKVHalf;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t kk = (k & 3) * 32;
                    umma_bf16_ss(tmem + qt * 256, umma_desc_sw128(qb + (k >> 2) * kQHalf + kk, 16, 1024),
                                 umma_desc_sw128(kb + (k >> 2) * kKVHalf + kk, 16, 1024), idesc_qk, k > 0 ? 1u : 0u);
                }
                umma_commit(&qbars[4 * qt + 0]);
            };
            auto issue_pv = [&](int qt, int g, bool first) {
                const uint32_t ts = tmem + qt * 256;
                const uint32_t vb = sv + (g % VST) * 2 * kKVHalf;
#pragma unroll
                for (int k = 0; k < kN / 16; ++k) {
                    umma_bf16_ts(ts + 128, ts + k * 8, umma_desc_sw128(vb + k * 16 * 128, kKVHalf, 1024), idesc_pv,
                                 (!first || k > 0) ? 1u : 0u);
                }
                umma_commit(&qbars[4 * qt + 2]);
            };
            bool ok = true;
            int gt = 0, nit = 0;
            // per query-tile slot (scalars, so that nothing goes to local memory): tiles so far (S, P and P.V
            // phases) and items so far (o_free phases)
            int cntA = 0, cntB = 0, nitA = 0, nitB = 0;
            for (;;) {
                if (!mbar_wait_bounded(&it_full[nit % IR], (nit / IR) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const volatile int* sp = item_slot + (nit % IR) * kSlotInts;
                const int item = sp[0];
                Item it;
                if (item >= 0) get_item(sp, it);
                mbar_arrive(&it_empty[nit % IR]);  // after the slot's last read
                if (item < 0) break;
                const int nA = it.nA, nB = it.nB;
                ok = mbar_wait_bounded(q_full, nit & 1, abort_flag) &&
                     mbar_wait_bounded(&k_full[gt % KST], (gt / KST) & 1, abort_flag);
#pragma unroll
                for (int qt = 0; qt < kQT; ++qt) {
                    if (!ok || qt >= it.nqt) continue;
                    const int cnt = qt == 0 ? cntA : cntB;
                    // S goes over the columns the slot's last P was read from
                    if (cnt > 0 && !mbar_wait_bounded(&qbars[4 * qt + 2], (cnt - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    issue_qk(qt, gt);
                }
                if (!ok) break;
                umma_commit(&k_empty[gt % KST]);
                if (it.ntiles == 1) umma_commit(q_empty);
                for (int j = 0; j < it.ntiles && ok; ++j) {
                    const int g = gt + j;
                    if (!mbar_wait_bounded(&v_full[g % VST], (g / VST) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int qt = 0; qt < kQT; ++qt) {
                        const int need = qt == 0 ? nA : nB;
                        const int cnt = qt == 0 ? cntA : cntB;
                        const int nitq = qt == 0 ? nitA : nitB;
                        if (!ok || j >= need) continue;
                        if (!mbar_wait_bounded(&qbars[4 * qt + 1], (cnt + j) & 1, abort_flag) ||  // P(j) written
                            (j == 0 && nitq > 0 &&
                             !mbar_wait_bounded(&qbars[4 * qt + 3], (nitq - 1) & 1, abort_flag))) {  // O read out
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        issue_pv(qt, g, j == 0);
                        if (j + 1 < need) {
                            // S(j+1) goes over the columns P(j) is read from: after P.V(j) has finished
                            if (!mbar_wait_bounded(&k_full[(g + 1) % KST], ((g + 1) / KST) & 1, abort_flag) ||
                                !mbar_wait_bounded(&qbars[4 * qt + 2], (cnt + j) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after_sync();
                            issue_qk(qt, g + 1);
                        }
                    }
                    if (!ok) break;
                    umma_commit(&v_empty[g % VST]);
                    if (j + 1 < it.ntiles) umma_commit(&k_empty[(g + 1) % KST]);
                    if (j + 2 == it.ntiles) umma_commit(q_empty);  // the item's last Q.K^T went out in this step
                }
                cntA += nA;
                ++nitA;
                if (it.nqt > 1) {
                    cntB += nB;
                    ++nitB;
                }
                gt += it.ntiles;
                ++nit;
                if (!ok) break;
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
        uint64_t* s_full = &qbars[4 * qt + 0];
        uint64_t* p_full = &qbars[4 * qt + 1];
        uint64_t* o_done = &qbars[4 * qt + 2];
        uint64_t* o_free = &qbars[4 * qt + 3];
        const int pair_bar = 1 + qt * 4 + (warp & 3);
        const uint32_t tmem_s = tmem + qt * 256;
        const uint32_t tmem_o = tmem_s + 128;
        const int t_local = r / G;
        const int g = r % G;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float sl = a.scale_log2;
        const float masked = sl >= 0.f ? -INFINITY : INFINITY;
        constexpr int NC = 2;  // 32-key chunks per half
        bool ok = true;
        int cnt = 0;  // tiles of this slot so far
        int xc = 0;   // exchanges with the other half so far (the buffer alternates)
        auto xslot = [&](int par, int h) -> float* { return xch + ((par * kQT + qt) * 2 + h) * 128 + r; };
        for (int k = 0;; ++k) {
            const bool got = ok && mbar_wait_warp(&it_full[k % IR], (k / IR) & 1, abort_flag);
            const volatile int* slot_k = item_slot + (k % IR) * kSlotInts;  // held until this item is done
            const int item = got ? slot_k[0] : -1;
            __syncwarp();
            // the two warps of a row pair leave together: a warp whose wait failed stops its partner too
            if (!pair_sync_and(pair_bar, got && item >= 0)) {
                if (!got || item >= 0) ok = false;
                break;
            }
            int ntq, lim, jz;  // tiles of this slot, this row's last key, the key tile past the context (or -1)
            {
                Item it;
                get_item(slot_k, it);
                ntq = qt == 0 ? it.nA : it.nB;
                const int tq = it.t_lo0 + qt * T + t_local;
                lim = (t_local < T && tq < it.n) ? (it.L - it.n + tq) : -1;
                jz = (it.L % kN != 0 && (it.L - 1) / kN < ntq) ? (it.L - 1) / kN : -1;
            }
            if (ntq == 0) {
                if (lane == 0) mbar_arrive(&it_empty[k % IR]);
                continue;
            }
            float m_used = -INFINITY, l = 0.f;
            for (int j = 0; j < ntq; ++j) {
                // a failed wait is carried to the pair barrier below, where both warps leave together
                const bool ok_s = ok && mbar_wait_warp(s_full, (cnt + j) & 1, abort_flag);
                tc_fence_after_sync();
                uint32_t sr[NC][32];
#pragma unroll
                for (int c = 0; c < NC; ++c) tmem_ld32(tmem_s + lane_base + half * 64 + c * 32, sr[c]);
                tmem_wait_ld();
                const int kv0 = j * kN + half * 64;
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
                // swap the partial maxima; the barrier also orders this half's S reads before the other half's
                // P stores over S's first 64 columns
                *xslot(xc & 1, half) = m0;
                tc_fence_before_sync();
                const bool pair_ok = pair_sync_and(pair_bar, ok_s);
                ++xc;
                if (!pair_ok) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const float other = *xslot((xc - 1) & 1, half ^ 1);
                const float mraw = sl >= 0.f ? fmaxf(m0, other) : fminf(m0, other);
                const float mx = mraw == masked ? -INFINITY : mraw * sl;
                const float m_new = fmaxf(m_used, mx);
                const bool rescale = m_used != -INFINITY && m_new > m_used + (float)kLazyRescale;
                const bool rescale_warp = __any_sync(0xffffffffu, rescale) != 0;
                const float alpha = rescale ? fast_exp2(m_used - m_new) : 1.f;
                if (rescale || m_used == -INFINITY) m_used = m_new;
                const float mref = m_used == -INFINITY ? 0.f : m_used;
                float rs0 = 0.f, rs1 = 0.f, rs2 = 0.f, rs3 = 0.f;
                const uint64_t slp = pack2f(sl, sl), mrp = pack2f(-mref, -mref);
#pragma unroll
                for (int c = 0; c < NC; ++c) {
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        float x0, x1;
                        ffma2(x0, x1, sr[c][2 * e2], sr[c][2 * e2 + 1], slp, mrp);
                        float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
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
                if (j == jz) {
                    // rows past the context: their P is 0, and 0 must not meet a NaN left in the pool
                    const int gv = slot_k[1] + j;
                    const bool v_ok = mbar_wait_warp(&v_full[gv % VST], (gv / VST) & 1, abort_flag);
                    if (!v_ok) ok = false;
                    const int first = max(0, slot_k[7] - j * kN);
                    const int chunks = v_ok ? (kN - first) * 16 : 0;
                    for (int i = t256; i < chunks; i += 256) {
                        const int row = first + (i >> 4);
                        const int h = (i >> 3) & 1;
                        *reinterpret_cast<uint4*>(smem + OFF_V + (gv % VST) * 2 * kKVHalf + h * kKVHalf + row * 128 +
                                                  (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full);
            }
            // the output's place, read before the slot is released (the producer may then refill it)
            Item it;
            get_item(slot_k, it);
            const int tq = it.t_lo0 + qt * T + t_local;
            const bool valid_row = t_local < T && tq < it.n;
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                                 ((size_t)(it.q0 + tq) * a.num_heads + (size_t)it.kvh * G + g) * kD + half * 64;
            __syncwarp();
            // both warps of the pair always get here, with the same number of exchanges behind them
            const bool ok_o = ok && mbar_wait_warp(o_done, (cnt + ntq - 1) & 1, abort_flag);
            if (lane == 0) mbar_arrive(&it_empty[k % IR]);
            *xslot(xc & 1, half) = l;
            const bool all_ok = pair_sync_and(pair_bar, ok_o);
            ++xc;
            if (!all_ok) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            l += *xslot((xc - 1) & 1, half ^ 1);
            const float inv = l > 0.f ? 1.f / l : 0.f;
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
            // O may now take the slot's next item
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
            cnt += ntq;
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
    static std::atomic<int> sm_count[64] = {};
    int sms = sm_count[dev & 63].load();
    if (sms == 0) {
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        sm_count[dev & 63].store(sms);
    }
    const int npairs = (max_query_len + kQT * T - 1) / (kQT * T);
    const long long nitems = (long long)npairs * a.num_seqs * a.num_kv_heads;
    if (nitems > INT32_MAX) return cudaErrorInvalidValue;
    const int grid = a.sched ? (int)std::min<long long>(nitems, sms) : (int)nitems;
    prefill_tc_kernel<G><<<grid, kThreads, kSmem, stream>>>(a, tq, tk, tv, npairs);
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
