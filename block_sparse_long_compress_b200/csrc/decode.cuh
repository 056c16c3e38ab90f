// Step 5 (decode) -- one query token per sequence attends to its selected
// key blocks (the QSA attention term of the per-token cost decomposition on
// page "Qwen4 in llama.cpp: Dissecting PR #27742", section "What Should Be
// Optimized After Correctness": indexed K/V gather over the selected cells).
//
// HBM-bound: every selected 64-token block is read once (K + V, 2*64*d
// bf16 = 32 KiB at d = 128).  The k selected slots of a (sequence, group)
// row are split over P CTAs (P <= 8) that form one thread-block cluster.
// Each CTA runs NW consumer warps; warp w owns one shared-memory stage and
// walks the CTA's slots w, w+NW, ...:
//     wait K(i) -> S = q K^T -> TMA K(i+1) into the freed K region ->
//     softmax (online, per head) -> wait V(i) -> O += P V -> TMA V(i+1)
// so the next block's loads overlap the current block's math.  S = q K^T
// and O = P V are bf16 mma.sync m16n8k16 tiles with fp32 accumulation: the
// G query heads of the group fill rows 0..G-1 of the 16-row A tile, K and V
// fragments come from the TMA tiles (128-byte swizzle) by ldmatrix /
// ldmatrix.trans, and P is reused from the S accumulators as the A
// fragment.  The warps' (max, sum, O) are merged in shared memory; the
// cluster's CTAs are merged by the leader CTA through distributed shared
// memory, which writes o.  No global workspace, no atomics.
#pragma once
#include <cooperative_groups.h>

#include "device.cuh"

namespace qsa {

template <int D>
struct DecodeCfg {
    static constexpr int NH = D / 64;
    static constexpr int HALF_BYTES = 64 * 128;
    static constexpr int KV_BYTES = 64 * D * 2;
    static constexpr int NW = 6;                       // consumer warps per CTA
    static constexpr int PART_FLOATS = 16 + 8 * D;     // m[8], l[8], O[8][D]
    static constexpr int SMEM_BYTES = NW * 2 * KV_BYTES + NW * PART_FLOATS * 4 + 1024;
    static constexpr int MAX_CLUSTER = 8;
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

template <int D, int G>
__global__ void __launch_bounds__(DecodeCfg<D>::NW * 32, 1) decode_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ idx,
    __nv_bfloat16 *__restrict__ o, int Hq, int Hkv, int L, int T_kv_max, int topk, int spc,
    float sm_scale_log2)
{
    using C = DecodeCfg<D>;
    constexpr int NW = C::NW;
    constexpr int PF = C::PART_FLOATS;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t bar_k[NW], bar_v[NW];
    __shared__ int abort_flag;
    __shared__ float cta_part[PF];   // this CTA's merged (m, l, O), read by the cluster leader

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *part = reinterpret_cast<float *>(smem + NW * 2 * C::KV_BYTES);   // [NW][PF]

    const int split = blockIdx.x;
    const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot1 = min(split * spc + spc, topk);
    const int last_blk = (L - 1) / 64;
    const int32_t *row_idx = idx + (long)bg * topk;
    const int kv_row0 = bg * T_kv_max;       // host checks B*Hkv*T_kv_max < 2^31

    uint8_t *ks = smem + warp * 2 * C::KV_BYTES;
    uint8_t *vs = ks + C::KV_BYTES;
    if (threadIdx.x == 0) abort_flag = 0;
    if (lane == 0) {
        mbar_init(&bar_k[warp], 1);
        mbar_init(&bar_v[warp], 1);
        fence_barrier_init();
    }
    __syncthreads();

    // block id of slot s of this CTA's range (-1 past the selection)
    auto block_of = [&](int s) -> int {
        if (s >= slot1) return -1;
        int j = __ldg(row_idx + s);
        if (j > last_blk) {
            if (lane == 0) report(QSA_ERR_BOUNDS, 3);
            j = -1;
        }
        return j;
    };
    auto load_k = [&](int j) {
        mbar_arrive_expect_tx(&bar_k[warp], C::KV_BYTES);
#pragma unroll
        for (int h = 0; h < C::NH; h++)
            tma_load_2d(ks + h * C::HALF_BYTES, &tmK, &bar_k[warp], h * 64, kv_row0 + 64 * j);
    };
    auto load_v = [&](int j) {
        mbar_arrive_expect_tx(&bar_v[warp], C::KV_BYTES);
#pragma unroll
        for (int h = 0; h < C::NH; h++)
            tma_load_2d(vs + h * C::HALF_BYTES, &tmV, &bar_v[warp], h * 64, kv_row0 + 64 * j);
    };

    int s = split * spc + warp;
    int j = block_of(s);
    if (lane == 0 && j >= 0) {
        load_k(j);
        load_v(j);
    }

    // query fragment: row = lane/4 = head within the group (rows >= G and
    // 8..15 are zero), columns 16ks + 2(lane%4) + {0,1} and +8.
    const int hr = lane >> 2, qc = (lane & 3) * 2;
    uint32_t qa[D / 16][2];
    {
        const __nv_bfloat16 *qrow = q + ((long)b * Hq + g * G + (hr < G ? hr : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; kk++) {
            const uint32_t lo = *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + qc);
            const uint32_t hi = *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 8 + qc);
            qa[kk][0] = hr < G ? lo : 0u;
            qa[kk][1] = hr < G ? hi : 0u;
        }
    }

    float m_run = -INFINITY, l_run = 0.f;
    float oacc[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; nt++) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;

    const uint32_t kaddr = smem_u32(ks), vaddr = smem_u32(vs);
    const int mi = lane >> 3, rr = lane & 7;
    uint32_t phase = 0;
    while (j >= 0) {
        const int s_next = s + NW;
        const int j_next = block_of(s_next);
        if (!mbar_wait(&bar_k[warp], phase, &abort_flag, 40)) break;
        // ---- S = q K^T (ldmatrix.x4: matrix mi = (k-step kk + (mi>>1), half mi&1))
        float sacc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; nt++) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; nt++) {
#pragma unroll
            for (int kk = 0; kk < D / 16; kk += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kaddr + sw128_offset(8 * nt + rr, 2 * (kk + (mi >> 1)) + (mi & 1)), b0, b1, b2, b3);
                mma_bf16_16816(sacc[nt], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
                mma_bf16_16816(sacc[nt], qa[kk + 1][0], 0u, qa[kk + 1][1], 0u, b2, b3);
            }
        }
        // K region consumed: prefetch the next block's keys
        __syncwarp();
        if (lane == 0 && j_next >= 0) {
            fence_proxy_async_smem();
            load_k(j_next);
        }
        // ---- online softmax (per head = per lane quad)
        const int lim = (L - 1) - 64 * j;    // keys c <= lim are visible
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; nt++) {
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int key = 8 * nt + qc + e;
                sacc[nt][e] = key <= lim ? sacc[nt][e] * sm_scale_log2 : -INFINITY;
                mx = fmaxf(mx, sacc[nt][e]);
            }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = fast_exp2(m_run - m_new);   // 0 on the first block
        m_run = m_new;
        l_run *= alpha;
#pragma unroll
        for (int nt = 0; nt < D / 8; nt++) {
            oacc[nt][0] *= alpha;
            oacc[nt][1] *= alpha;
        }
        uint32_t pa[8];
#pragma unroll
        for (int nt = 0; nt < 8; nt++) {
            const float p0 = fast_exp2(sacc[nt][0] - m_run), p1 = fast_exp2(sacc[nt][1] - m_run);
            l_run += p0 + p1;
            pa[nt] = pack_bf16x2(p0, p1);
        }
        // ---- O += P V (ldmatrix.trans: matrix mi = (keys half mi&1, column tile nt + (mi>>1)))
        if (!mbar_wait(&bar_v[warp], phase, &abort_flag, 41)) break;
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
        __syncwarp();
        if (lane == 0 && j_next >= 0) {
            fence_proxy_async_smem();
            load_v(j_next);
        }
        phase ^= 1u;
        s = s_next;
        j = j_next;
    }
    // row sums of the warp: reduce the quad's partial sums
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

    // ---- merge the warps of this CTA in shared memory
    float *wp = part + warp * PF;
    if ((lane & 3) == 0) {
        wp[hr] = m_run;
        wp[8 + hr] = l_run;
    }
#pragma unroll
    for (int nt = 0; nt < D / 8; nt++) {
        wp[16 + hr * D + 8 * nt + qc] = oacc[nt][0];
        wp[16 + hr * D + 8 * nt + qc + 1] = oacc[nt][1];
    }
    __syncthreads();
    // CTA partial (shifted by the CTA max, unnormalised)
    for (int e = threadIdx.x; e < G * D; e += NW * 32) {
        const int h = e / D, c = e % D;
        float mc = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; w++) mc = fmaxf(mc, part[w * PF + h]);
        float oc = 0.f, lc = 0.f;
        if (mc != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; w++) {
                const float f = fast_exp2(part[w * PF + h] - mc);
                oc += f * part[w * PF + 16 + h * D + c];
                lc += f * part[w * PF + 8 + h];
            }
        }
        cta_part[16 + h * D + c] = oc;
        if (c == 0) {
            cta_part[h] = mc;
            cta_part[8 + h] = lc;
        }
    }
    // ---- merge the cluster's CTAs (one per split) through distributed shared memory
    cluster.sync();
    if (cluster.block_rank() == 0) {
        const int P = (int)cluster.num_blocks();
        for (int e = threadIdx.x; e < G * D; e += NW * 32) {
            const int h = e / D, c = e % D;
            float mc = -INFINITY;
            for (int r = 0; r < P; r++) {
                const float *rp = cluster.map_shared_rank(cta_part, r);
                mc = fmaxf(mc, rp[h]);
            }
            float oc = 0.f, lc = 0.f;
            if (mc != -INFINITY) {
                for (int r = 0; r < P; r++) {
                    const float *rp = cluster.map_shared_rank(cta_part, r);
                    const float f = fast_exp2(rp[h] - mc);
                    oc += f * rp[16 + h * D + c];
                    lc += f * rp[8 + h];
                }
            }
            o[((long)b * Hq + g * G + h) * D + c] = __float2bfloat16_rn(lc > 0.f ? oc / lc : 0.f);
        }
    }
    cluster.sync();   // the other CTAs' shared memory must outlive the leader's reads
}

}  // namespace qsa
