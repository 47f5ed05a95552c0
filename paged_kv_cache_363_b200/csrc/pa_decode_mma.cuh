// Tensor-core consumer of the paged decode kernel: bf16 with a group of 2, 4 or 8
// query heads per kv head.  The group's query heads times a block's 16 tokens
// times head_dim is a dense tile, so both contractions run as warp-level bf16 MMAs
// (m16n8k16, fp32 accumulation):
//   S[16 tokens][8 heads]   = K_tile . q^T      tokens on M, heads on N, head_dim on K
//   O^T[head_dim][8 heads] += V_tile^T . P      head_dim on M, heads on N, tokens on K
// The S accumulator becomes the P operand in registers (an 8x8 transpose per half,
// movmatrix).  P is split into a bf16 head and a bf16 remainder and both are
// multiplied, so the weights keep about 16 mantissa bits and the products with
// the bf16 V values accumulate in fp32 like the CUDA-core path.
//
// Operands come from K/V tiles written by 2-D TMA tensor copies with the 128-byte
// swizzle: 16-byte chunk c of row r of a 64-column box sits at r*128 + (c ^ r%8)*16,
// which makes every ldmatrix below free of bank conflicts.  Tokens past the
// context get -inf logits and zeroed V rows (the pool may hold anything there).
#pragma once

#include "pa_decode_common.cuh"

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

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D_, int B_, int G_>
struct MmaConsumer {
    using T = __nv_bfloat16;
    static constexpr int D = D_, B = B_, G = G_;
    static constexpr bool kTensorLoads = true;  // 2-D TMA boxes of 64 columns, 128-byte swizzle
    static constexpr int HALF_BYTES = B * 128;  // one 64-column box of a tile
    static constexpr int NHALF = D / 64;
    static constexpr int DK = D / 16;           // k-steps of K . q^T
    static constexpr int DM = D / 16;           // m-tiles of V^T . P
    static constexpr int SUB = B / 16;          // 16-token sub-tiles per block
    static constexpr int SCRATCH_FLOATS = 0;

    static_assert(D % 64 == 0 && B % 16 == 0, "tile shape");
    static_assert(G >= 1 && G <= 8, "at most 8 heads on the MMA N side");
    static_assert(HALF_BYTES % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");

    uint32_t qb[DK][2];  // q^T as the B operand: k = head_dim, n = head g
    float o[DM][4];      // O^T accumulators: rows mt*16+g (+8), heads 2t, 2t+1
    float m0, m1;        // running max of heads 2t, 2t+1 (base-2 logits)
    float l0, l1;        // this lane's share of their softmax sums
    float sl;
    int lane, g, t, i8, k_row, v_row, j8;

    __device__ __forceinline__ void init(float*, int lane_)
    {
        lane = lane_;
        g = lane >> 2;
        t = lane & 3;
        j8 = lane >> 3;            // which 8x8 matrix of an ldmatrix.x4 this lane addresses
        i8 = lane & 7;             // its row inside that matrix; also the swizzle key (row % 8)
        k_row = (j8 & 1) * 8 + i8; // token row (within 16) this lane addresses for K
        v_row = (j8 >> 1) * 8 + i8;
    }

    __device__ __forceinline__ void begin_unit(const T* q_smem, float scale_log2)
    {
        const uint32_t* qp = reinterpret_cast<const uint32_t*>(q_smem);
#pragma unroll
        for (int kk = 0; kk < DK; ++kk) {
            qb[kk][0] = g < G ? qp[(g * D + kk * 16 + 2 * t) / 2] : 0u;
            qb[kk][1] = g < G ? qp[(g * D + kk * 16 + 2 * t + 8) / 2] : 0u;
        }
#pragma unroll
        for (int mt = 0; mt < DM; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
        sl = scale_log2;
    }

    __device__ __forceinline__ void block(const unsigned char* kt_, unsigned char* vt_, int nvalid)
    {
        const uint32_t kt = smem_u32(kt_);
        const uint32_t vt = smem_u32(vt_);
        if (nvalid < B) {
            // tokens past the context: zero their V rows so 0-weights meet finite values
            const int n16 = (B - nvalid) * NHALF * 8;
            for (int idx = lane; idx < n16; idx += 32) {
                const int r = nvalid + idx / (NHALF * 8);
                const int rem = idx % (NHALF * 8);
                *reinterpret_cast<uint4*>(vt_ + (rem >> 3) * HALF_BYTES + r * 128 + (rem & 7) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
#pragma unroll
        for (int sub = 0; sub < SUB; ++sub) {
            if (sub * 16 >= nvalid) break;
            // ---- S = K . q^T for 16 tokens
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < DK; ++kk) {
                const int chunk = kk * 2 + (j8 >> 1);
                const uint32_t addr =
                    kt + (chunk >> 3) * HALF_BYTES + (sub * 16 + k_row) * 128 + (((chunk & 7) ^ i8) << 4);
                uint32_t af[4];
                ldsm_x4(af, addr);
                mma_bf16(sc, af, qb[kk][0], qb[kk][1]);
            }
            const int tok0 = sub * 16 + g;
            float s0 = sc[0] * sl, s1 = sc[1] * sl, s2 = sc[2] * sl, s3 = sc[3] * sl;
            if (tok0 >= nvalid) s0 = s1 = -INFINITY;
            if (tok0 + 8 >= nvalid) s2 = s3 = -INFINITY;
            // ---- online softmax over the sub-tile (max across the 16 token rows of each head)
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
            for (int mt = 0; mt < DM; ++mt) {
                o[mt][0] *= al0;
                o[mt][1] *= al1;
                o[mt][2] *= al0;
                o[mt][3] *= al1;
            }
            // ---- P as the B operand: bf16 head + bf16 remainder, transposed 8x8 halves
            const uint32_t h01 = pack_bf16(p0, p1);
            const uint32_t h23 = pack_bf16(p2, p3);
            const uint32_t r01 =
                pack_bf16(p0 - __uint_as_float(h01 << 16), p1 - __uint_as_float(h01 & 0xffff0000u));
            const uint32_t r23 =
                pack_bf16(p2 - __uint_as_float(h23 << 16), p3 - __uint_as_float(h23 & 0xffff0000u));
            const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
            const uint32_t bl0 = movmatrix_trans(r01), bl1 = movmatrix_trans(r23);
            // ---- O^T += V^T . P
#pragma unroll
            for (int mt = 0; mt < DM; ++mt) {
                const int chunk = mt * 2 + (j8 & 1);
                const uint32_t addr =
                    vt + (chunk >> 3) * HALF_BYTES + (sub * 16 + v_row) * 128 + (((chunk & 7) ^ i8) << 4);
                uint32_t af[4];
                ldsm_x4_trans(af, addr);
                mma_bf16(o[mt], af, bh0, bh1);
                mma_bf16(o[mt], af, bl0, bl1);
            }
        }
        // the zeroing above wrote a TMA destination through the generic proxy
        if (nvalid < B) fence_proxy_async_smem();
    }

    __device__ __forceinline__ void end_unit(float* mg_m, float* mg_l, float* mg_acc, int warp)
    {
        float la = l0, lb = l1;
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            la += __shfl_xor_sync(0xffffffffu, la, off);
            lb += __shfl_xor_sync(0xffffffffu, lb, off);
        }
        const int h0 = 2 * t, h1 = 2 * t + 1;
        if (g == 0) {
            if (h0 < G) {
                mg_m[warp * G + h0] = m0;
                mg_l[warp * G + h0] = la;
            }
            if (h1 < G) {
                mg_m[warp * G + h1] = m1;
                mg_l[warp * G + h1] = lb;
            }
        }
#pragma unroll
        for (int mt = 0; mt < DM; ++mt) {
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
};

}  // namespace
}  // namespace pa
