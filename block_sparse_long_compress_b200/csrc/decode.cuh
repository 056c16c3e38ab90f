// Step 5 (decode) -- one query token per sequence attends to its selected
// key blocks (the QSA attention term of the per-token cost decomposition on
// page "Qwen4 in llama.cpp: Dissecting PR #27742", section "What Should Be
// Optimized After Correctness": indexed K/V gather over the selected cells).
//
// HBM-bound: every selected 64-token block is read once (K + V, 2*64*d
// bf16).  Split-K: CTA (split, b*Hkv+g) owns NW consecutive slots of the
// row's selection; warp w loads block slot (split*NW + w) with two TMA
// boxes per tensor (128-byte swizzle) and computes, for the G query heads
// of the group (padded to the 16 rows of an m16n8k16 tile),
//     S = q K^T   (bf16 mma.sync, fp32 accumulate; B fragments by ldmatrix)
//     P = exp2(S*c - m), l = sum P
//     O = P V     (P re-used from the S accumulators as the A fragment;
//                  V fragments by ldmatrix.trans)
// The warps' (m, l, O) are merged in shared memory, written to the
// workspace, and the last CTA of each (b, g) to finish (atomic ticket, no
// waiting) merges all splits and writes o.  These contractions are tiny
// (G rows); tensor cores are used only to keep the FMA pipes off the
// critical path of an HBM-bound stream.
#pragma once
#include "device.cuh"

namespace qsa {

template <int D>
struct DecodeCfg {
    static constexpr int NH = D / 64;
    static constexpr int HALF_BYTES = 64 * 128;
    static constexpr int KV_BYTES = 64 * D * 2;
    static constexpr int WARP_BYTES = 2 * KV_BYTES;   // K + V of one block
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk c16 (0 .. D/8-1) of tile row `row` in a
// 64-row tile stored as D/64 TMA boxes of 64 x 128 B with 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_offset(int row, int c16)
{
    return (uint32_t)((c16 >> 3) * (64 * 128) + row * 128 + (((c16 & 7) ^ (row & 7)) << 4));
}

struct DecodePartial {
    float *m;   // [B*Hkv][nsplit][8]
    float *l;   // [B*Hkv][nsplit][8]
    float *o;   // [B*Hkv][nsplit][8][D]
    int *ticket;  // [B*Hkv]
};

template <int D, int G, int NW>
__global__ void __launch_bounds__(NW * 32) decode_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ idx,
    __nv_bfloat16 *__restrict__ o, DecodePartial part, int Hq, int Hkv, int L, int T_kv_max,
    int topk, float sm_scale_log2)
{
    using C = DecodeCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t bar[NW];
    __shared__ float red_m[NW][8], red_l[NW][8];
    __shared__ float red_o[NW][8][D];
    __shared__ int is_last;
    __shared__ int abort_flag;

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int split = blockIdx.x, nsplit = gridDim.x;
    const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = split * NW + warp;
    const int last_blk = (L - 1) / 64;
    int j = slot < topk ? idx[(long)bg * topk + slot] : -1;
    if (j > last_blk) {
        report(QSA_ERR_BOUNDS, 3);
        j = -1;
    }
    uint8_t *ks = smem + warp * C::WARP_BYTES;
    uint8_t *vs = ks + C::KV_BYTES;
    if (threadIdx.x == 0) abort_flag = 0;
    if (lane == 0) {
        mbar_init(&bar[warp], 1);
        fence_barrier_init();
        if (j >= 0) {
            const int y = (int)((long)bg * T_kv_max + 64L * j);
            mbar_arrive_expect_tx(&bar[warp], C::WARP_BYTES);
#pragma unroll
            for (int h = 0; h < C::NH; h++) {
                tma_load_2d(ks + h * C::HALF_BYTES, &tmK, &bar[warp], h * 64, y);
                tma_load_2d(vs + h * C::HALF_BYTES, &tmV, &bar[warp], h * 64, y);
            }
        }
    }
    __syncthreads();

    // query fragment: row = lane/4 = head within the group (rows >= G and
    // 8..15 are zero), columns 16ks + 2(lane%4) + {0,1} and +8.
    const int hr = lane >> 2, qc = (lane & 3) * 2;
    uint32_t qa[D / 16][2];
    {
        const __nv_bfloat16 *qrow = q + ((long)b * Hq + g * G + (hr < G ? hr : 0)) * D;
#pragma unroll
        for (int ks_ = 0; ks_ < D / 16; ks_++) {
            uint32_t lo = *reinterpret_cast<const uint32_t *>(qrow + 16 * ks_ + qc);
            uint32_t hi = *reinterpret_cast<const uint32_t *>(qrow + 16 * ks_ + 8 + qc);
            qa[ks_][0] = hr < G ? lo : 0u;
            qa[ks_][1] = hr < G ? hi : 0u;
        }
    }

    float m = -INFINITY, l = 0.f;
    float oacc[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; nt++) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;

    if (j >= 0 && mbar_wait(&bar[warp], 0, &abort_flag, 40)) {
        const uint32_t kaddr = smem_u32(ks), vaddr = smem_u32(vs);
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; nt++) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        // S = q K^T: matrix mi of ldmatrix.x4 = (k-step ks_ + (mi>>1), half mi&1)
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int nt = 0; nt < 8; nt++) {
#pragma unroll
            for (int ks_ = 0; ks_ < D / 16; ks_ += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kaddr + sw128_offset(8 * nt + rr, 2 * (ks_ + (mi >> 1)) + (mi & 1)), b0, b1, b2, b3);
                mma_bf16_16816(s[nt], qa[ks_][0], 0u, qa[ks_][1], 0u, b0, b1);
                mma_bf16_16816(s[nt], qa[ks_ + 1][0], 0u, qa[ks_ + 1][1], 0u, b2, b3);
            }
        }
        // mask keys after the query position, then the block max per head
        const int lim = (L - 1) - 64 * j;
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; nt++) {
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int key = 8 * nt + qc + e;
                s[nt][e] = key <= lim ? s[nt][e] * sm_scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[nt][e]);
            }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        m = mx;
        uint32_t pa[8];
#pragma unroll
        for (int nt = 0; nt < 8; nt++) {
            const float p0 = fast_exp2(s[nt][0] - m), p1 = fast_exp2(s[nt][1] - m);
            l += p0 + p1;
            pa[nt] = pack_bf16x2(p0, p1);
        }
        // O = P V: ldmatrix.trans matrix mi = (keys half mi&1, column tile nt + (mi>>1))
#pragma unroll
        for (int k2 = 0; k2 < 4; k2++) {
#pragma unroll
            for (int nt = 0; nt < D / 8; nt += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vaddr + sw128_offset(16 * k2 + 8 * (mi & 1) + rr, nt + (mi >> 1)), b0, b1, b2, b3);
                mma_bf16_16816(oacc[nt], pa[2 * k2], 0u, pa[2 * k2 + 1], 0u, b0, b1);
                mma_bf16_16816(oacc[nt + 1], pa[2 * k2], 0u, pa[2 * k2 + 1], 0u, b2, b3);
            }
        }
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
    }

    // ---- merge the warps of this CTA
    if ((lane & 3) == 0) {
        red_m[warp][hr] = m;
        red_l[warp][hr] = l;
    }
#pragma unroll
    for (int nt = 0; nt < D / 8; nt++) {
        red_o[warp][hr][8 * nt + qc] = oacc[nt][0];
        red_o[warp][hr][8 * nt + qc + 1] = oacc[nt][1];
    }
    __syncthreads();
    const long pbase = (long)bg * nsplit + split;
    for (int e = threadIdx.x; e < G * D; e += NW * 32) {
        const int h = e / D, c = e % D;
        float mc = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; w++) mc = fmaxf(mc, red_m[w][h]);
        float oc = 0.f, lc = 0.f;
        if (mc != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; w++) {
                const float f = fast_exp2(red_m[w][h] - mc);
                oc += f * red_o[w][h][c];
                lc += f * red_l[w][h];
            }
        }
        part.o[(pbase * 8 + h) * D + c] = oc;
        if (c == 0) {
            part.m[pbase * 8 + h] = mc;
            part.l[pbase * 8 + h] = lc;
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(&part.ticket[bg], 1) == nsplit - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // ---- last CTA of (b, g): merge all splits
    for (int e = threadIdx.x; e < G * D; e += NW * 32) {
        const int h = e / D, c = e % D;
        float mc = -INFINITY;
        for (int s_ = 0; s_ < nsplit; s_++) mc = fmaxf(mc, __ldcg(part.m + ((long)bg * nsplit + s_) * 8 + h));
        float oc = 0.f, lc = 0.f;
        if (mc != -INFINITY) {
            for (int s_ = 0; s_ < nsplit; s_++) {
                const long pb = (long)bg * nsplit + s_;
                const float f = fast_exp2(__ldcg(part.m + pb * 8 + h) - mc);
                oc += f * __ldcg(part.o + (pb * 8 + h) * D + c);
                lc += f * __ldcg(part.l + pb * 8 + h);
            }
        }
        o[((long)b * Hq + g * G + h) * D + c] = __float2bfloat16_rn(lc > 0.f ? oc / lc : 0.f);
    }
    if (threadIdx.x == 0) part.ticket[bg] = 0;   // ready for the next call
}

}  // namespace qsa
