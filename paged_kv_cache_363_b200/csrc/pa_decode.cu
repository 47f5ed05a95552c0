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
//  * Work units are (sequence, context partition, kv head).  All query heads of the
//    kv head's group are packed into one unit, so each K/V byte leaves HBM once.
//  * A plan kernel lists the (sequence, partition) pairs longest first; a persistent
//    kernel (a few CTAs per SM) takes units from that list with an atomic counter, so
//    the grid holds no empty CTAs and the short units are the ones left at the end.
//  * In each CTA one warp fetches units ahead of use (block-table slice and q into a
//    small shared ring), one thread streams the units' K/V tiles into a ring of
//    shared-memory stages with the TMA engine (1-D bulk copies of whole tiles, or 2-D
//    tensor boxes with the 128-byte swizzle for the tensor-core consumer; each CTA
//    loads its own tiles) and four consumer warps take alternate blocks.  The stream of tiles
//    runs across unit boundaries, so the pipeline does not drain between units.
//  * Consumers: CUDA cores (fp32; bf16 with one query head per kv head) or tensor
//    cores (bf16 with 2, 4 or 8 query heads per kv head); see the two policy headers.
//  * At the end of a unit each warp leaves its softmax state in shared memory and goes
//    on with the next unit; the warp that consumed the unit's last tile merges the four
//    states.  A sequence longer than one partition leaves (max, sum, unnormalised
//    output) per partition in the workspace and a log-sum-exp merge kernel combines
//    them.  Plan, persistent and merge kernels are chained with programmatic dependent
//    launch.
//  * The first wave of CTAs does not wait for the plan: when the partition length is
//    fixed, CTA b starts on partition 0 of sequence b / Hkv (kv head b % Hkv), which
//    the plan lists at position b / Hkv, while the plan kernel still runs.
//  * Logits are kept in base-2 units (q pre-scaled by scale*log2 e) and exponentials
//    use exp2f, the reformulation of online softmax by Milakov & Gimelshein (2018).
//  * Every wait is bounded: a wait that runs out raises PA_DEV_WAIT_TIMEOUT and the
//    CTA winds down instead of hanging.  Bad block indices or context lengths raise a
//    status bit and are clamped instead of being dereferenced.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "pa_decode_common.cuh"
#include "pa_decode_fma.cuh"
#include "pa_decode_mma.cuh"
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {

// ---------------------------------------------------------------- tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

unsigned long long current_context_id()
{
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// The pool [num_blocks][kv_heads][B][D] as a 2-D bf16 tensor of rows of D elements;
// boxes of 64 columns x `B` rows (one stage tile), 128-byte swizzle.  A small cache avoids re-encoding
// the maps of the same pools on every call.
cudaError_t tensor_map(CUtensorMap* out, const void* pool, uint64_t rows, int D, int B)
{
    struct Entry {
        const void* ptr;
        uint64_t rows;
        int d, b, dev;
        CUtensorMap map;
    };
    static std::mutex mu;
    static Entry cache[16] = {};
    static int next = 0;
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return ce;
    {
        std::lock_guard<std::mutex> lk(mu);
        for (auto& en : cache)
            if (en.ptr == pool && en.rows == rows && en.d == D && en.b == B && en.dev == dev) {
                *out = en.map;
                return cudaSuccess;
            }
    }
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap m;
    std::memset(&m, 0, sizeof(m));
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)B};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pool), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    std::lock_guard<std::mutex> lk(mu);
    Entry& en = cache[next];
    next = (next + 1) % 16;
    en.ptr = pool;
    en.rows = rows;
    en.d = D;
    en.b = B;
    en.dev = dev;
    en.map = m;
    *out = m;
    return cudaSuccess;
}

namespace {

constexpr int kEndUnit = 1;    // no more work for this CTA
constexpr int kSplitUnit = 2;  // the sequence spans several partitions

struct UnitInfo {
    int s, kvh, part, nb, b0, first, L, flags, np, pad[3];
};

// Shared-memory budget of one CTA: two CTAs per SM, each with about 96 KB of K/V
// stages in flight, keep enough bytes moving to cover the HBM latency under load.
constexpr int kCtaSmemBudget = 110 * 1024;

// Cons: the consumer policy (tiles of Cons::B = 16 tokens); BS: the physical block
// size.  A stage holds one 16-token tile of K and of V; a block of BS tokens is
// BS / 16 consecutive tiles.
template <class Cons, int BS>
struct Persist {
    using T = typename Cons::T;
    static constexpr int D = Cons::D, G = Cons::G;
    static constexpr int TR = Cons::B;                  // tokens per stage
    static constexpr int SPB = BS / TR;                 // stages per physical block
    static constexpr int TILE_BYTES = TR * D * (int)sizeof(T);
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K tile, then V tile
    static constexpr int NCW = 4;                       // consumer warps
    static constexpr int UR = 2;                        // units held: the current one and the next
    static constexpr int MAX_PBLK = kMaxPartitionTokens / 16;
    static constexpr int QBYTES = G * D * (int)sizeof(T);
    static constexpr int SLOT_BYTES = (QBYTES + MAX_PBLK * 4 + (int)sizeof(UnitInfo) + 127) / 128 * 128;
    static constexpr int THREADS = (NCW + 2) * 32;      // consumers, tile producer, unit producer
    static constexpr int MERGE_FLOATS = NCW * G * (D + 2);
    static constexpr int NBAR_FIXED = 3 * UR + 2;
    static constexpr int FIXED_BYTES = UR * SLOT_BYTES + MERGE_FLOATS * 4 + NCW * Cons::SCRATCH_FLOATS * 4 +
                                       NBAR_FIXED * 8 + 16 + 1024;
    // Stage i of the CTA's stream is consumed by warp i % NCW.  With NSTAGES a multiple
    // of NCW the warp that waits for a stage's n-th fill also consumed its (n-1)-th, so
    // a one-bit phase parity is never stale.
    static constexpr int NSTAGES =
        cmax(NCW, cmin(24, ((kCtaSmemBudget - FIXED_BYTES - 16 * 24) / STAGE_BYTES) / NCW * NCW));
    static constexpr int OFF_SLOT = NSTAGES * STAGE_BYTES;
    static constexpr int OFF_MERGE = OFF_SLOT + UR * SLOT_BYTES;
    static constexpr int OFF_SCRATCH = OFF_MERGE + MERGE_FLOATS * 4;
    static constexpr int OFF_BAR = (OFF_SCRATCH + NCW * Cons::SCRATCH_FLOATS * 4 + 7) / 8 * 8;
    static constexpr int NBAR = 2 * NSTAGES + NBAR_FIXED;
    static constexpr int OFF_ABORT = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_ABORT + 16 + 1024;  // + slack to align the base to 1024 bytes

    static_assert(BS % TR == 0, "block size must be a multiple of the stage tile");
    static_assert(NSTAGES % NCW == 0, "stage ring must be a multiple of the consumer warps");
    static_assert(TILE_BYTES % 1024 == 0, "tiles keep the 1024-byte alignment of the swizzle atoms");
    static_assert(QBYTES % 16 == 0, "q rows are bulk-copied");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// Moves 16-token tile h of one physical block's K and V into a stage; completion is
// counted on bar.
template <class Cons, int BS>
__device__ __forceinline__ void issue_tile(unsigned char* stage, const DecodeArgs& a, const CUtensorMap* tk,
                                           const CUtensorMap* tv, int phys, int kvh, int h, uint64_t* bar,
                                           uint64_t policy)
{
    using P = Persist<Cons, BS>;
    mbar_arrive_expect_tx(bar, 2 * P::TILE_BYTES);
    if constexpr (Cons::kTensorLoads) {
        const int row = (phys * a.num_kv_heads + kvh) * BS + h * P::TR;
        const uint32_t dk = smem_u32(stage);
#pragma unroll
        for (int hh = 0; hh < Cons::NHALF; ++hh) {
            tma_load_2d(dk + hh * Cons::HALF_BYTES, tk, hh * 64, row, bar, policy);
            tma_load_2d(dk + P::TILE_BYTES + hh * Cons::HALF_BYTES, tv, hh * 64, row, bar, policy);
        }
    } else {
        const size_t off = (((size_t)phys * a.num_kv_heads + kvh) * BS + (size_t)h * P::TR) * P::D * sizeof(typename P::T);
        bulk_g2s_hint(stage, static_cast<const unsigned char*>(a.k_cache) + off, P::TILE_BYTES, bar, policy);
        bulk_g2s_hint(stage + P::TILE_BYTES, static_cast<const unsigned char*>(a.v_cache) + off, P::TILE_BYTES,
                      bar, policy);
    }
}

template <class Cons, int BS>
__global__ void __launch_bounds__(Persist<Cons, BS>::THREADS, 2)
    decode_persistent_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                             const __grid_constant__ CUtensorMap tmap_v)
{
    using P = Persist<Cons, BS>;
    using T = typename Cons::T;
    constexpr int D = P::D, B = BS, G = P::G, NCW = P::NCW, NS = P::NSTAGES, UR = P::UR, TR = P::TR,
                  SPB = P::SPB;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
    uint64_t* full = bars;            // stage filled (tx bytes)
    uint64_t* empty = bars + NS;      // stage consumed
    uint64_t* ufull = bars + 2 * NS;  // unit slot filled (q bytes)
    uint64_t* uempty = ufull + UR;    // unit slot released (consumers and tile producer)
    uint64_t* utab = uempty + UR;     // unit slot's block-table slice written (tile producer)
    uint64_t* mg_full = utab + UR;    // every consumer warp's state of the unit is in the merge buffer
    uint64_t* mg_free = mg_full + 1;  // the unit's finish has read the merge buffer
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P::OFF_ABORT);
    float* mg_m = reinterpret_cast<float*>(smem + P::OFF_MERGE);
    float* mg_l = mg_m + NCW * G;
    float* mg_acc = mg_l + NCW * G;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int st = 0; st < NS; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        for (int u = 0; u < UR; ++u) {
            mbar_init(&ufull[u], 1);
            mbar_init(&uempty[u], 2);
            mbar_init(&utab[u], 1);
        }
        mbar_init(mg_full, NCW);
        mbar_init(mg_free, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // A CTA of the first wave starts on its own unit while the plan kernel still runs:
    // only its unit producer waits for the plan, before its second unit.  Every other
    // CTA waits here; the plan kernel's list and counters are visible after the wait.
    const bool early = (int)blockIdx.x < a.first_wave;
    if (!early) pdl_wait_primary();

    auto slot = [&](int k) { return smem + P::OFF_SLOT + (k % UR) * P::SLOT_BYTES; };
    auto slot_table = [&](int k) { return reinterpret_cast<int*>(slot(k) + P::QBYTES); };
    auto slot_info = [&](int k) { return reinterpret_cast<UnitInfo*>(slot(k) + P::QBYTES + P::MAX_PBLK * 4); };

    if (warp == NCW + 1) {
        // ---------------- unit producer: takes units from the plan, fills the unit ring
        // The first unit's list entry is requested together with the pair count, not
        // after it: its index is inside the list whatever the count (the grid has at
        // most one CTA per unit the list can hold).  A first-wave CTA knows its first
        // unit without the list: partition 0 of sequence b / Hkv (the plan puts that
        // pair at list position b / Hkv).
        unsigned nunits = 0;
        uint2 e_first;
        auto plan_ready = [&]() { nunits = __ldcg(a.plan + 1) * (unsigned)a.num_kv_heads; };
        if (early) {
            const int s0 = (int)(blockIdx.x / (unsigned)a.num_kv_heads);
            e_first = make_uint2((unsigned)s0 << 11, (unsigned)clamped_context(a, s0, B, false));
        } else {
            e_first = __ldcg(a.plan_list + blockIdx.x / (unsigned)a.num_kv_heads);
            plan_ready();
        }
        // This CTA takes no more units.  The last CTA to stop (at the end marker or on
        // a wait that gave up) resets the work counter, so the plan in the workspace
        // serves the next run as it is (one plan per decode step, one run per layer);
        // it happens while the CTAs still finish their last units, off the kernel's
        // critical path.  Lane 0 only.
        auto leave = [&]() {
            if (atomicAdd(a.plan + 4, 1u) == gridDim.x - 1) {
                a.plan[0] = 0u;
                a.plan[4] = 0u;
            }
        };
        int first = 0;
        int k = 0;
        bool ended = false;
        for (;; ++k) {
            if (k >= UR && !mbar_wait_warp(&uempty[k % UR], ((k / UR) & 1) ^ 1, abort_flag)) {
                if (lane == 0) {
                    atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                    leave();
                }
                *abort_flag = 1;
                break;
            }
            UnitInfo* info = slot_info(k);
            // the first unit of CTA b is unit b; later ones come from the counter
            unsigned u = blockIdx.x;
            if (k > 0) {
                if (k == 1 && early) {
                    pdl_wait_primary();
                    plan_ready();
                }
                if (lane == 0) u = gridDim.x + atomicAdd(a.plan, 1u);
                u = __shfl_sync(0xffffffffu, u, 0);
            }
            if (u >= nunits && !(k == 0 && early)) {
                if (lane == 0) {
                    info->flags = kEndUnit;
                    mbar_arrive(&utab[k % UR]);
                    mbar_arrive(&ufull[k % UR]);
                    leave();
                }
                ended = true;
                break;
            }
            const uint2 e = k == 0 ? e_first : a.plan_list[u / (unsigned)a.num_kv_heads];
            const int kvh = (int)(u % (unsigned)a.num_kv_heads);
            const int s = (int)(e.x >> 11);
            const int part = (int)(e.x & 2047u);
            const int L = (int)e.y;
            const int nblk_seq = (L + B - 1) / B;
            const int pb = (k == 0 && early) ? a.partition_blocks : (int)a.plan[2];  // equal when early
            const int b0 = part * pb;
            const int nb = max(0, min(pb, nblk_seq - b0));
            int* tab = slot_table(k);
            // A first-wave unit reads its table slice (partition 0: the row's first pb
            // entries, all inside the row) in the same trip to memory as its context
            // length, not after it; entries past the context are loaded but never used.
            const int nload = (k == 0 && early) ? min(pb, a.max_blocks_per_seq) : nb;
            for (int i = lane; i < nload; i += 32)
                tab[i] = __ldg(a.block_tables + (size_t)s * a.max_blocks_per_seq + b0 + i);
            if (lane == 0) {
                info->s = s;
                info->kvh = kvh;
                info->part = part;
                info->nb = nb;
                info->b0 = b0;
                info->first = first;
                info->L = L;
                info->flags = nblk_seq > pb ? kSplitUnit : 0;
                info->np = (nblk_seq + pb - 1) / pb;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&utab[k % UR]);  // the tile producer may start on this unit
                mbar_arrive_expect_tx(&ufull[k % UR], P::QBYTES);
                bulk_g2s(slot(k), static_cast<const T*>(a.q) + ((size_t)s * a.num_heads + (size_t)kvh * G) * D,
                         P::QBYTES, &ufull[k % UR]);
            }
            first += nb * SPB;
        }
        // No q copy may still be landing in shared memory at exit: wait for the fills of
        // the last units.  After an end marker, slot k % UR has moved on past unit k - UR
        // (a parity wait on that older phase would alias), so only units k-UR+1 .. k-1.
        if (lane == 0) {
            volatile int never = 0;
            const int j0 = k - UR + (ended ? 1 : 0);
            for (int j = j0 < 0 ? 0 : j0; j < k; ++j)
                if (!mbar_wait_bounded(&ufull[j % UR], (j / UR) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else if (warp == NCW) {
        // ---------------- tile producer: one thread streams K/V tiles into the stages
        if (lane == 0) {
            const uint64_t policy = policy_evict_first();
            int i = 0;  // blocks issued so far (the CTA's stream index)
            bool ok = true;
            for (int k = 0; ok; ++k) {
                if (!mbar_wait_bounded(&utab[k % UR], (k / UR) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const UnitInfo* info = slot_info(k);
                if (info->flags & kEndUnit) break;
                const int nt = info->nb * SPB;
                const int kvh = info->kvh;
                const int* tab = slot_table(k);
                int phys = 0;
                for (int j = 0; j < nt; ++j, ++i) {
                    const int st = i % NS;
                    if (i >= NS && !mbar_wait_bounded(&empty[st], ((i / NS) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (j % SPB == 0) {
                        phys = tab[j / SPB];
                        if ((unsigned)phys >= (unsigned)a.num_blocks) {
                            atomicOr(a.status, PA_DEV_BAD_BLOCK);
                            phys = 0;
                        }
                    }
                    issue_tile<Cons, BS>(smem + st * P::STAGE_BYTES, a, &tmap_k, &tmap_v, phys, kvh, j % SPB,
                                         &full[st], policy);
                }
                // done with this unit's table: the slot may be refilled once the consumers are done too
                if (ok) mbar_arrive(&uempty[k % UR]);
            }
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // no tile copy may still be landing in shared memory at exit
            volatile int never = 0;
            for (int j = i - NS < 0 ? 0 : i - NS; j < i; ++j)
                if (!mbar_wait_bounded(&full[j % NS], (j / NS) & 1, &never)) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else {
        // ---------------- consumers
        // At a unit's end each warp puts its state in the merge buffer and moves on to
        // the next unit without waiting.  The warp that consumed the unit's last tile
        // (usually the last to get there) waits for the other states, merges them and
        // writes the result, then frees the buffer and the unit slot.  A warp may write
        // its state for unit k only after the finish of unit k-1 has freed the buffer,
        // so arrivals on mg_full for unit k all belong to phase k, and one-bit parities
        // on both barriers are never stale.
        Cons cons;
        cons.init(reinterpret_cast<float*>(smem + P::OFF_SCRATCH) + warp * Cons::SCRATCH_FLOATS, lane);
        bool ok = true;
        for (int k = 0; ok; ++k) {
            if (!mbar_wait_bounded(&ufull[k % UR], (k / UR) & 1, abort_flag)) {
                ok = false;
                break;
            }
            const UnitInfo* info = slot_info(k);
            if (info->flags & kEndUnit) break;
            const int first = info->first, nt = info->nb * SPB, L = info->L;
            const int tok0 = info->b0 * B;  // first token of the unit
            cons.begin_unit(reinterpret_cast<const T*>(slot(k)), a.scale_log2);
            for (int i = first + ((warp - first % NCW) + NCW) % NCW; i < first + nt; i += NCW) {
                const int st = i % NS;
                if (!mbar_wait_bounded(&full[st], (i / NS) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                unsigned char* stage = smem + st * P::STAGE_BYTES;
                cons.block(stage, stage + P::TILE_BYTES, min(TR, L - tok0 - (i - first) * TR));
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
            if (!ok) break;
            if (k > 0 && !mbar_wait_bounded(mg_free, (k - 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            cons.end_unit(mg_m, mg_l, mg_acc, warp);
            __syncwarp();
            if (lane == 0) mbar_arrive(mg_full);
            const int finisher = ((first + nt - 1) % NCW + NCW) % NCW;
            if (warp == finisher) {
                if (!mbar_wait_bounded(mg_full, k & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const bool split = (info->flags & kSplitUnit) != 0;
                finish_unit_warp<T, D, G, NCW>(a, mg_m, mg_l, mg_acc, info->s, info->kvh, info->part, split,
                                               first % NCW, lane);
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(mg_free);
                    mbar_arrive(&uempty[k % UR]);
                }
            }
        }
        if (!ok) {
            if (lane == 0) atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
        }
    }
}

// ---------------------------------------------------------------- launch

// CTAs of the persistent kernel resident on the current device at once (cached per device).
template <class Cons, int BS>
cudaError_t resident_ctas(int* out)
{
    using P = Persist<Cons, BS>;
    static std::atomic<int> cached[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int d = dev & 63;
    int v = cached[d].load();
    if (v == 0) {
        e = cudaFuncSetAttribute(decode_persistent_kernel<Cons, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 P::SMEM);
        if (e != cudaSuccess) return e;
        int occ = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_persistent_kernel<Cons, BS>, P::THREADS,
                                                          P::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        v = (occ < 1 ? 1 : occ) * sms;
        cached[d].store(v);
    }
    *out = v;
    return cudaSuccess;
}

template <class Cons, int BS>
cudaError_t launch_persistent(const DecodeArgs& a, cudaStream_t stream)
{
    using P = Persist<Cons, BS>;
    CUtensorMap tk, tv;
    std::memset(&tk, 0, sizeof(tk));
    std::memset(&tv, 0, sizeof(tv));
    if constexpr (Cons::kTensorLoads) {
        if (a.phases & kDecodeRun) {
            const uint64_t rows = (uint64_t)a.num_blocks * a.num_kv_heads * BS;
            cudaError_t e = tensor_map(&tk, a.k_cache, rows, P::D, P::TR);
            if (e != cudaSuccess) return e;
            e = tensor_map(&tv, a.v_cache, rows, P::D, P::TR);
            if (e != cudaSuccess) return e;
        }
    }
    int ctas = 0;
    cudaError_t e = resident_ctas<Cons, BS>(&ctas);
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)a.num_kv_heads * a.num_seqs * a.num_partitions;
    const unsigned grid = (unsigned)(units < ctas ? units : ctas);
    DecodeArgs args = a;
    args.num_ctas = (int)grid;
    // An automatic partition starts at 1024 tokens instead of 512 when units twice as long still balance and
    // halving the partitions saves merge work: at least three (sequence, kv head) pairs per CTA with a context
    // bound of 3072 tokens or more (long sequences split into half as many partitions), or at least ten pairs
    // per CTA (many sequences just over one partition).  Plan and run calls take the same arguments, so they
    // make the same choice.
    const int64_t pairs_all = (int64_t)a.num_seqs * a.num_kv_heads;
    if (a.adaptive && a.partition_blocks * BS == 512 &&
        ((pairs_all >= 3LL * grid && a.max_context_len >= 3072) || pairs_all >= 10LL * grid))
        args.partition_blocks = 1024 / BS;
    // The first wave: with the partition fixed, CTA b < first_wave starts on kv head
    // b % Hkv of partition 0 of sequence b / Hkv without waiting for the plan.  The plan
    // grows an automatic partition only when the tokens of all sequences exceed
    // 4 x partition x CTAs, which the bound num_seqs x max_context_len rules out here.
    const bool fixed_partition =
        !a.adaptive || (int64_t)a.num_seqs * a.max_context_len <= 4LL * args.partition_blocks * BS * (int64_t)grid;
    const int64_t pairs0 = (int64_t)a.num_seqs * a.num_kv_heads;
    args.first_wave = fixed_partition ? (int)(pairs0 < (int64_t)grid ? pairs0 : (int64_t)grid) : 0;

    if (a.phases & kDecodePlan) {
        // one CTA; fewer threads for small batches keep its barriers short
        const int plan_threads = a.num_seqs <= 256 ? 256 : (a.num_seqs <= 512 ? 512 : 1024);
        decode_plan_kernel<<<1, plan_threads, 0, stream>>>(args, BS);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (!(a.phases & kDecodeRun)) return cudaSuccess;
    e = launch_pdl(decode_persistent_kernel<Cons, BS>, dim3(grid), dim3(P::THREADS), (size_t)P::SMEM, stream, args,
                   tk, tv);
    if (e != cudaSuccess || a.num_partitions <= 1) return e;
    return launch_merge<typename Cons::T, P::D>(args, BS, stream);
}

template <typename T, int D, int B>
cudaError_t dispatch_group(const DecodeArgs& a, int group, cudaStream_t stream)
{
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        switch (group) {
            case 1: return launch_persistent<FmaConsumer<T, D, 16, 1>, B>(a, stream);
            case 2: return launch_persistent<MmaConsumer<D, 16, 2>, B>(a, stream);
            case 4: return launch_persistent<MmaConsumer<D, 16, 4>, B>(a, stream);
            case 8: return launch_persistent<MmaConsumer<D, 16, 8>, B>(a, stream);
            default: return cudaErrorInvalidValue;
        }
    } else {
        switch (group) {
            case 1: return launch_persistent<FmaConsumer<T, D, 16, 1>, B>(a, stream);
            case 2: return launch_persistent<FmaConsumer<T, D, 16, 2>, B>(a, stream);
            case 4: return launch_persistent<FmaConsumer<T, D, 16, 4>, B>(a, stream);
            case 8: return launch_persistent<FmaConsumer<T, D, 16, 8>, B>(a, stream);
            default: return cudaErrorInvalidValue;
        }
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

bool decode_uses_tensor_cores(pa_dtype dtype, int head_dim, int group)
{
    return dtype == PA_DTYPE_BF16 && (head_dim == 64 || head_dim == 128) && (group == 2 || group == 4 || group == 8);
}

cudaError_t launch_decode(const DecodeArgs& a, pa_dtype dtype, int head_dim, int block_size, int group,
                          cudaStream_t stream)
{
    if (dtype == PA_DTYPE_F32) return dispatch_dim<float>(a, head_dim, block_size, group, stream);
    return dispatch_dim<__nv_bfloat16>(a, head_dim, block_size, group, stream);
}

}  // namespace pa
