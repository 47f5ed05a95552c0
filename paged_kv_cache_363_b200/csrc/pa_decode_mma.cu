// Paged decode attention for grouped-query heads (bf16, group of 2, 4 or 8 query
// heads per kv head) on the tensor cores of sm_100a.
//
// Same computation and work split as the CUDA-core kernel (one CTA per kv head,
// sequence and context partition; "PagedAttention and vLLM Architecture",
// section 2: walk the block table, q.K per gathered block, online softmax across
// blocks fused with the product by the V blocks).  The group's query heads times a
// block's 16 tokens times head_dim is a dense tile, so the two contractions run as
// warp-level bf16 MMAs (m16n8k16, fp32 accumulation):
//   S[16 tokens][8 heads]    = K_tile . q^T      tokens on M, heads on N, head_dim on K
//   O^T[head_dim][8 heads]  += V_tile^T . P      head_dim on M, heads on N, tokens on K
// The S accumulator becomes the P operand in registers (one 8x8 transpose per
// half, movmatrix).  P is split into a bf16 head and a bf16 remainder and both are
// multiplied, so the weights keep about 16 mantissa bits: the products with the
// bf16 V values are then accumulated in fp32 like the CUDA-core path.
//
// Operand staging: the producer thread loads each physical block's K and V tiles
// with 2-D TMA tensor copies (two 64-column boxes per tile, 128-byte swizzle, no
// multicast), so the ldmatrix reads of both operands are free of bank conflicts.
// Masked tokens of a sequence's last block get -inf logits and zeroed V rows (the
// pool may hold anything there).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "pa_decode_common.cuh"
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {

namespace {

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// c += a . b  (m16n8k16, bf16 inputs, fp32 accumulators)
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Two fp32 values to a bf16 pair (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D, int B, int G>
struct MmaCfg {
    static constexpr int TILE_BYTES = B * D * 2;
    static constexpr int HALF_BYTES = B * 128;            // one 64-column swizzled box of a tile
    static constexpr int NHALF = D / 64;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int NCW = 4;                          // consumer warps
    // Stage i % NSTAGES holds block i, consumed by warp i % NCW; NSTAGES a multiple
    // of NCW keeps every mbarrier phase wait unambiguous (see the CUDA-core kernel).
    static constexpr int NSTAGES = cmax(NCW, cmin(8, 65536 / STAGE_BYTES));
    static constexpr int THREADS = (NCW + 1) * 32;
    static constexpr int DK = D / 16;                      // k-steps of K . q^T
    static constexpr int DM = D / 16;                      // m-tiles of V^T . P
    static constexpr int SUB = B / 16;                     // 16-token sub-tiles per block
    static constexpr int MAX_PBLK = kMaxPartitionTokens / 16;
    static constexpr int OFF_BAR = NSTAGES * STAGE_BYTES;  // from the 1024-byte aligned base
    static constexpr int OFF_TABLE = OFF_BAR + 2 * NSTAGES * 8;
    static constexpr int OFF_ABORT = OFF_TABLE + MAX_PBLK * 4;
    static constexpr int SMEM = OFF_ABORT + 16 + 1024;     // + slack to align the base
    static constexpr int MERGE_BYTES = NCW * G * (D + 2) * 4;

    static_assert(D % 64 == 0 && B % 16 == 0, "tile shape");
    static_assert(G >= 1 && G <= 8, "at most 8 heads on the MMA N side");
    static_assert(NSTAGES % NCW == 0, "stage ring must be a multiple of the consumer warps");
    static_assert(MERGE_BYTES <= OFF_BAR, "merge area must fit in the stage ring");
    static_assert(HALF_BYTES % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <int D, int B, int G>
__global__ void __launch_bounds__(MmaCfg<D, B, G>::THREADS, 3)
    decode_partition_mma_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                                const __grid_constant__ CUtensorMap tmap_v)
{
    using C = MmaCfg<D, B, G>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    unsigned char* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t base = smem_u32(smem);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty_bar = full_bar + C::NSTAGES;
    int* s_table = reinterpret_cast<int*>(smem + C::OFF_TABLE);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);

    const int kvh = blockIdx.x;
    const int s = blockIdx.y;
    const int part = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

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

    const int g = lane >> 2;   // MMA row group: token (S) or head_dim row (O^T)
    const int t = lane & 3;    // MMA column pair: heads 2t, 2t+1
    float m0 = -INFINITY, m1 = -INFINITY;  // running max of heads 2t, 2t+1 (base-2 logits)
    float l0 = 0.f, l1 = 0.f;              // this lane's share of their softmax sums
    float o[C::DM][4];                     // O^T accumulators: rows mt*16+g (+8), heads 2t, 2t+1
#pragma unroll
    for (int mt = 0; mt < C::DM; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    if (warp == C::NCW) {
        // ---------------- producer: one thread issues the TMA tile loads
        if (lane == 0) {
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
                const int row = (phys * a.num_kv_heads + kvh) * B;
                const uint32_t dk = base + st * C::STAGE_BYTES;
                const uint32_t dv = dk + C::TILE_BYTES;
                mbar_arrive_expect_tx(&full_bar[st], 2 * C::TILE_BYTES);
#pragma unroll
                for (int hh = 0; hh < C::NHALF; ++hh) {
                    tma_load_2d(dk + hh * C::HALF_BYTES, &tmap_k, hh * 64, row, &full_bar[st], policy);
                    tma_load_2d(dv + hh * C::HALF_BYTES, &tmap_v, hh * 64, row, &full_bar[st], policy);
                }
                ++issued;
            }
            if (!ok) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *s_abort = 1;
            }
            volatile int never = 0;
            for (int i = max(0, issued - C::NSTAGES); i < issued; ++i)
                if (!mbar_wait_bounded(&full_bar[i % C::NSTAGES], (i / C::NSTAGES) & 1, &never))
                    atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
        }
    } else {
        // ---------------- consumers: one block per warp at a time, all on MMAs
        uint32_t qb[C::DK][2];  // q^T as the B operand: k = head_dim, n = head g
        {
            const uint32_t* qp = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                                   ((size_t)s * a.num_heads + (size_t)kvh * G) * D);
#pragma unroll
            for (int kk = 0; kk < C::DK; ++kk) {
                qb[kk][0] = g < G ? __ldg(qp + (g * D + kk * 16 + 2 * t) / 2) : 0u;
                qb[kk][1] = g < G ? __ldg(qp + (g * D + kk * 16 + 2 * t + 8) / 2) : 0u;
            }
        }
        const float sl = a.scale_log2;
        const int j8 = lane >> 3;  // which 8x8 matrix of an ldmatrix.x4 this lane addresses
        const int i8 = lane & 7;   // its row inside that matrix; also the swizzle key (row % 8)
        // row offsets (tokens) inside a 16-token sub-tile for the K and V loads
        const int k_row = (j8 & 1) * 8 + i8;
        const int v_row = (j8 >> 1) * 8 + i8;

        for (int i = warp; i < nblk; i += C::NCW) {
            const int st = i % C::NSTAGES;
            if (!mbar_wait_bounded(&full_bar[st], (i / C::NSTAGES) & 1, s_abort)) {
                atomicOr(a.status, PA_DEV_WAIT_TIMEOUT);
                *s_abort = 1;
                break;
            }
            const uint32_t kt = base + st * C::STAGE_BYTES;
            const uint32_t vt = kt + C::TILE_BYTES;
            const int nvalid = min(B, L - (b0 + i) * B);
            if (nvalid < B) {
                // tokens past the context: zero their V rows so 0-weights meet finite values
                unsigned char* vrow = smem + st * C::STAGE_BYTES + C::TILE_BYTES;
                const int n16 = (B - nvalid) * C::NHALF * 8;
                for (int idx = lane; idx < n16; idx += 32) {
                    const int r = nvalid + idx / (C::NHALF * 8);
                    const int rem = idx % (C::NHALF * 8);
                    *reinterpret_cast<uint4*>(vrow + (rem >> 3) * C::HALF_BYTES + r * 128 + (rem & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                __syncwarp();
            }

#pragma unroll
            for (int sub = 0; sub < C::SUB; ++sub) {
                if (sub * 16 >= nvalid) break;
                // ---- S = K . q^T for 16 tokens
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < C::DK; ++kk) {
                    const int chunk = kk * 2 + (j8 >> 1);
                    const uint32_t addr = kt + (chunk >> 3) * C::HALF_BYTES + (sub * 16 + k_row) * 128 +
                                          (((chunk & 7) ^ i8) << 4);
                    uint32_t af[4];
                    ldsm_x4(af, addr);
                    mma_bf16(sc, af, qb[kk][0], qb[kk][1]);
                }
                const int tok0 = sub * 16 + g;
                float s0 = sc[0] * sl, s1 = sc[1] * sl, s2 = sc[2] * sl, s3 = sc[3] * sl;
                if (tok0 >= nvalid) s0 = s1 = -INFINITY;
                if (tok0 + 8 >= nvalid) s2 = s3 = -INFINITY;
                // ---- online softmax over the sub-tile (max across the 8 token rows of each head)
                float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
                m0 = mn0;
                m1 = mn1;
                const float p0 = exp2f(s0 - mn0), p1 = exp2f(s1 - mn1);
                const float p2 = exp2f(s2 - mn0), p3 = exp2f(s3 - mn1);
                l0 = fmaf(l0, al0, p0 + p2);
                l1 = fmaf(l1, al1, p1 + p3);
#pragma unroll
                for (int mt = 0; mt < C::DM; ++mt) {
                    o[mt][0] *= al0;
                    o[mt][1] *= al1;
                    o[mt][2] *= al0;
                    o[mt][3] *= al1;
                }
                // ---- P as the B operand: bf16 head + bf16 remainder, transposed 8x8 halves
                const uint32_t h01 = pack_bf16(p0, p1);
                const uint32_t h23 = pack_bf16(p2, p3);
                const uint32_t r01 = pack_bf16(p0 - __uint_as_float(h01 << 16), p1 - __uint_as_float(h01 & 0xffff0000u));
                const uint32_t r23 = pack_bf16(p2 - __uint_as_float(h23 << 16), p3 - __uint_as_float(h23 & 0xffff0000u));
                const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
                const uint32_t bl0 = movmatrix_trans(r01), bl1 = movmatrix_trans(r23);
                // ---- O^T += V^T . P
#pragma unroll
                for (int mt = 0; mt < C::DM; ++mt) {
                    const int chunk = mt * 2 + (j8 & 1);
                    const uint32_t addr = vt + (chunk >> 3) * C::HALF_BYTES + (sub * 16 + v_row) * 128 +
                                          (((chunk & 7) ^ i8) << 4);
                    uint32_t af[4];
                    ldsm_x4_trans(af, addr);
                    mma_bf16(o[mt], af, bh0, bh1);
                    mma_bf16(o[mt], af, bl0, bl1);
                }
            }
            // the zeroing above wrote a TMA destination through the generic proxy
            if (nvalid < B) fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
        // softmax sums: add the shares of the 8 lanes holding the same heads
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
    }

    __syncthreads();  // the stage ring is free: reuse it for the cross-warp merge

    float* mg_m = reinterpret_cast<float*>(smem);
    float* mg_l = mg_m + C::NCW * G;
    float* mg_acc = mg_l + C::NCW * G;
    if (warp < C::NCW) {
        const int h0 = 2 * t, h1 = 2 * t + 1;
        if (g == 0) {
            if (h0 < G) {
                mg_m[warp * G + h0] = m0;
                mg_l[warp * G + h0] = l0;
            }
            if (h1 < G) {
                mg_m[warp * G + h1] = m1;
                mg_l[warp * G + h1] = l1;
            }
        }
#pragma unroll
        for (int mt = 0; mt < C::DM; ++mt) {
            const int d = mt * 16 + g;
            if (h0 < G) {
                mg_acc[(warp * G + h0) * D + d] = o[mt][0];
                mg_acc[(warp * G + h0) * D + d + 8] = o[mt][2];
            }
            if (h1 < G) {
                mg_acc[(warp * G + h1) * D + d] = o[mt][1];
                mg_acc[(warp * G + h1) * D + d + 8] = o[mt][3];
            }
        }
    }
    __syncthreads();
    finish_partition<__nv_bfloat16, D, G, C::NCW, C::THREADS>(a, mg_m, mg_l, mg_acc, s, kvh, part, split);
}

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

// The pool [num_blocks][kv_heads][B][D] as a 2-D bf16 tensor of rows of D elements;
// boxes of 64 columns x B rows, 128-byte swizzle.  A small cache avoids re-encoding
// the maps of the same pools on every call.
struct MapCache {
    struct Entry {
        const void* ptr;
        uint64_t rows;
        int d, b, dev;
        CUtensorMap map;
    };
    std::mutex mu;
    Entry e[16] = {};
    int next = 0;
};

cudaError_t tensor_map(CUtensorMap* out, const void* pool, uint64_t rows, int D, int B)
{
    static MapCache cache;
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return ce;
    {
        std::lock_guard<std::mutex> lk(cache.mu);
        for (auto& en : cache.e)
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
    std::lock_guard<std::mutex> lk(cache.mu);
    MapCache::Entry& en = cache.e[cache.next];
    cache.next = (cache.next + 1) % 16;
    en.ptr = pool;
    en.rows = rows;
    en.d = D;
    en.b = B;
    en.dev = dev;
    en.map = m;
    *out = m;
    return cudaSuccess;
}

template <int D, int B, int G>
cudaError_t launch_mma_typed(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t stream)
{
    using C = MmaCfg<D, B, G>;
    static std::atomic<uint64_t> attr_set{0};
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) return e0;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(decode_partition_mma_kernel<D, B, G>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit);
    }
    dim3 grid(a.num_kv_heads, a.num_seqs, a.num_partitions);
    decode_partition_mma_kernel<D, B, G><<<grid, C::THREADS, C::SMEM, stream>>>(a, tk, tv);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.num_partitions <= 1) return e;
    return launch_merge<__nv_bfloat16, D>(a, B, stream);
}

template <int D, int B>
cudaError_t mma_group(const DecodeArgs& a, int group, const CUtensorMap& tk, const CUtensorMap& tv,
                      cudaStream_t stream)
{
    switch (group) {
        case 2: return launch_mma_typed<D, B, 2>(a, tk, tv, stream);
        case 4: return launch_mma_typed<D, B, 4>(a, tk, tv, stream);
        case 8: return launch_mma_typed<D, B, 8>(a, tk, tv, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool decode_uses_tensor_cores(pa_dtype dtype, int head_dim, int group)
{
    return dtype == PA_DTYPE_BF16 && (head_dim == 64 || head_dim == 128) && (group == 2 || group == 4 || group == 8);
}

cudaError_t launch_decode_mma(const DecodeArgs& a, int head_dim, int block_size, int group, cudaStream_t stream)
{
    const uint64_t rows = (uint64_t)a.num_blocks * a.num_kv_heads * block_size;
    CUtensorMap tk, tv;
    cudaError_t e = tensor_map(&tk, a.k_cache, rows, head_dim, block_size);
    if (e != cudaSuccess) return e;
    e = tensor_map(&tv, a.v_cache, rows, head_dim, block_size);
    if (e != cudaSuccess) return e;
    if (head_dim == 128) {
        if (block_size == 16) return mma_group<128, 16>(a, group, tk, tv, stream);
        if (block_size == 32) return mma_group<128, 32>(a, group, tk, tv, stream);
    } else if (head_dim == 64) {
        if (block_size == 16) return mma_group<64, 16>(a, group, tk, tv, stream);
        if (block_size == 32) return mma_group<64, 32>(a, group, tk, tv, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pa
