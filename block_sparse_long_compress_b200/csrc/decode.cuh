// Step 5 (decode) -- one query token per sequence attends to its selected
// key blocks (the QSA attention term of the per-token cost decomposition on
// page "Qwen4 in llama.cpp: Dissecting PR #27742", section "What Should Be
// Optimized After Correctness": indexed K/V gather over the selected cells).
//
// HBM-bound: every selected 64-token block is read once (K + V, 2*64*d
// bf16 = 32 KiB at d = 128) and the arithmetic per byte is tiny, so the
// kernel is built to keep enough bytes in flight on every SM.
//
// The k selected slots of a (sequence, group) row are split into P equal
// ranges, one per CTA; the row's P CTAs form one thread-block cluster
// (P <= 8) and two CTAs share an SM.  Per CTA:
//   producer warp   keeps a ring of NS stages full with TMA loads (one
//                   stage = one block's K and V, 128-byte swizzle),
//                   refilling a stage as soon as the consumers release it;
//   4 consumer warps  every warp takes 16 of each block's 64 keys:
//                   S^T = K q^T with the keys on the MMA M side (m16n8k16,
//                   the G heads of the group on N), online softmax per head
//                   over the warp's keys, P^T turned into the B operand by
//                   movmatrix, O^T += V^T P^T (d on M, V^T by
//                   ldmatrix.trans).  No padding rows: 16 MMAs per warp and
//                   block.
// The P x 4 warp partials (max, sum, O) of the row are merged in one pass
// through distributed shared memory, each CTA finishing 1/P of the row's
// outputs.  No global workspace, no global atomics.
//
// Caches are either contiguous ([B][Hkv][T_kv_max][d]; one length L for all
// sequences) or paged for serving: every sequence has its own length
// seq_lens[b], and its logical block j lives in page block_table[b][j] of
// [num_pages][Hkv][64][d] -- the cache-cell addresses the selector's indices
// are turned into.  Indices, lengths and pages are checked before any load
// (QSA_ERR_BOUNDS; the offending block is skipped).
#pragma once
#include <cooperative_groups.h>

#include "device.cuh"

namespace qsa {

template <int D>
struct DecodeCfg {
    static constexpr int NH = D / 64;                  // 64-column TMA boxes per row
    static constexpr int HALF_BYTES = 64 * 128;        // one 64-row x 128-byte box
    static constexpr int KV_BYTES = 64 * D * 2;        // one block's K (or V)
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int CTAS_PER_SM = 2;
    static constexpr int RING_BYTES = 96 * 1024;       // NS stages; two CTAs per SM
    static constexpr int NS = RING_BYTES / STAGE_BYTES;
    static constexpr int NC = 4;                       // consumer warps
    static constexpr int THREADS = (NC + 1) * 32;
    static constexpr int PART_FLOATS = 16 + 8 * D;     // m[8], l[8], O[8][D] of one warp
    static constexpr int SMEM_BYTES = RING_BYTES + 1024;
    static constexpr int MAX_SLOTS = 64;
    static constexpr int MAX_CLUSTER = 8;
    static_assert(NS >= 2, "ring too small");
    static_assert(NC * PART_FLOATS * 4 <= RING_BYTES, "merge scratch must fit in the ring");
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

// Transpose of an 8x8 b16 matrix held in the mma fragment layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a)
{
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
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
__global__ void __launch_bounds__(DecodeCfg<D>::THREADS, DecodeCfg<D>::CTAS_PER_SM) decode_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ idx,
    __nv_bfloat16 *__restrict__ o, int Hq, int Hkv, int L, int T_kv_max, int topk, int spc,
    float sm_scale_log2, const int32_t *__restrict__ seq_lens, const int32_t *__restrict__ block_table,
    int max_blocks, int num_pages)
{
    using C = DecodeCfg<D>;
    constexpr int NS = C::NS;
    constexpr int NC = C::NC;
    constexpr int PF = C::PART_FLOATS;
    constexpr int MAX_SRC = C::MAX_CLUSTER * NC;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full[NS], empty[NS];
    __shared__ int blocks[C::MAX_SLOTS];   // the CTA's valid block ids in slot order
    __shared__ int rows[C::MAX_SLOTS];     // and the first cache row of each (TMA coordinate)
    __shared__ int nb_sh, issued_sh, abort_flag;
    __shared__ float wgt[MAX_SRC][8];      // per-source, per-head merge weights
    __shared__ float lsrc[MAX_SRC][8];
    __shared__ float inv_l[8];

    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *part = reinterpret_cast<float *>(ring);   // after the loop: [NC][PF] warp partials

    const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int P = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kv_row0 = bg * T_kv_max;       // host checks B*Hkv*T_kv_max < 2^31

    // no global memory before the previous kernel on the stream (normally
    // the selection that writes idx) has completed
    grid_dependency_wait();
    grid_launch_dependents();
    // this sequence's cache length (the current token is its last position)
    int Lb = L;
    if (seq_lens) {
        Lb = __ldg(seq_lens + b);
        const long cap = block_table ? 64L * max_blocks : (long)T_kv_max;
        if (Lb < 1 || Lb > cap) {
            if (threadIdx.x == 0) report(QSA_ERR_BOUNDS, 6);
            Lb = 0;   // no block is valid: the row's output is zero
        }
    }
    const int last_blk = Lb > 0 ? (Lb - 1) / 64 : -1;
    // the CTA's valid block ids, compacted in slot order
    const int slot0 = rank * spc;
    const int slot1 = min(slot0 + spc, topk);
    if (warp == 0) {
        int n = 0;
        for (int base = slot0; base < slot1; base += 32) {
            const int s = base + lane;
            int j = s < slot1 ? __ldg(idx + (long)bg * topk + s) : -1;
            if (j > last_blk) {
                report(QSA_ERR_BOUNDS, 3);
                j = -1;
            }
            int row = 0;
            if (j >= 0) {
                if (block_table) {
                    const int page = __ldg(block_table + (long)b * max_blocks + j);
                    if (page < 0 || page >= num_pages) {
                        report(QSA_ERR_BOUNDS, 7);
                        j = -1;
                    } else {
                        row = (page * Hkv + g) * 64;   // host checks num_pages*Hkv*64 < 2^31
                    }
                } else {
                    row = kv_row0 + 64 * j;
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, j >= 0);
            if (j >= 0) {
                blocks[n + __popc(m & ((1u << lane) - 1u))] = j;
                rows[n + __popc(m & ((1u << lane) - 1u))] = row;
            }
            n += __popc(m);
        }
        if (lane == 0) nb_sh = n;
    }
    if (threadIdx.x == 32) {
        abort_flag = 0;
        issued_sh = 0;
#pragma unroll
        for (int s = 0; s < NS; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC);
        }
        fence_barrier_init();
    }
    __syncthreads();
    const int nb = nb_sh;

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float oacc[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; mt++) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;

    if (warp == NC) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int i = 0;
            for (; i < nb; i++) {
                const int st = i % NS;
                if (i >= NS) {
                    if (!mbar_wait(&empty[st], ((i / NS) - 1) & 1, &abort_flag, 42)) break;
                    fence_proxy_async_smem();
                }
                const int row = rows[i];
                mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
                uint8_t *ks = ring + st * C::STAGE_BYTES;
                uint8_t *vs = ks + C::KV_BYTES;
#pragma unroll
                for (int h = 0; h < C::NH; h++) tma_load_2d(ks + h * C::HALF_BYTES, &tmK, &full[st], h * 64, row);
#pragma unroll
                for (int h = 0; h < C::NH; h++) tma_load_2d(vs + h * C::HALF_BYTES, &tmV, &full[st], h * 64, row);
            }
            issued_sh = i;
        }
    } else {
        // ---------------------------------------------------- consumers
        // B operand of S^T = K q^T: column n = head lane/4 of the group
        // (zero for n >= G), rows k = d.
        const int hn = lane >> 2, qc = (lane & 3) * 2;
        uint32_t qb[D / 16][2];
        {
            const __nv_bfloat16 *qrow = q + ((long)b * Hq + g * G + (hn < G ? hn : 0)) * D;
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                const uint32_t lo = *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + qc);
                const uint32_t hi = *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 8 + qc);
                qb[kk][0] = hn < G ? lo : 0u;
                qb[kk][1] = hn < G ? hi : 0u;
            }
        }
        const int k0 = 16 * warp;                                  // the warp's keys in each block
        const int krow_a = k0 + (lane & 7) + 8 * ((lane >> 3) & 1);  // K rows for ldmatrix (A of S^T)
        const int kchunk_a = lane >> 4;
        const int vrow_a = k0 + (lane & 7) + 8 * (lane >> 4);        // V rows for ldmatrix.trans (A of O^T)
        const int vchunk_a = (lane >> 3) & 1;
        const int key_lo = k0 + (lane >> 2);                         // keys of this thread's S^T entries
        for (int i = 0; i < nb; i++) {
            const int st = i % NS;
            if (!mbar_wait(&full[st], (i / NS) & 1, &abort_flag, 40)) break;
            const int j = blocks[i];
            const uint32_t kaddr = smem_u32(ring + st * C::STAGE_BYTES);
            const uint32_t vaddr = kaddr + C::KV_BYTES;
            // ---- S^T (16 keys x 8 heads) = K q^T
            float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(kaddr + sw128_offset(krow_a, 2 * kk + kchunk_a), a0, a1, a2, a3);
                mma_bf16_16816(s, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
            }
            // ---- online softmax per head over the warp's keys
            const int lim = (Lb - 1) - 64 * j;   // keys c <= lim are visible
            const bool v0 = key_lo <= lim, v1 = key_lo + 8 <= lim;
            s[0] = v0 ? s[0] * sm_scale_log2 : -INFINITY;
            s[1] = v0 ? s[1] * sm_scale_log2 : -INFINITY;
            s[2] = v1 ? s[2] * sm_scale_log2 : -INFINITY;
            s[3] = v1 ? s[3] * sm_scale_log2 : -INFINITY;
            float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
            // a head whose keys are all masked so far keeps a finite reference
            const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
            const float al0 = fast_exp2(m_run[0] - mu0), al1 = fast_exp2(m_run[1] - mu1);
            m_run[0] = mn0;
            m_run[1] = mn1;
            const float p0 = fast_exp2(s[0] - mu0), p1 = fast_exp2(s[1] - mu1);
            const float p2 = fast_exp2(s[2] - mu0), p3 = fast_exp2(s[3] - mu1);
            l_run[0] = l_run[0] * al0 + (p0 + p2);
            l_run[1] = l_run[1] * al1 + (p1 + p3);
#pragma unroll
            for (int mt = 0; mt < D / 16; mt++) {
                oacc[mt][0] *= al0;
                oacc[mt][1] *= al1;
                oacc[mt][2] *= al0;
                oacc[mt][3] *= al1;
            }
            // P^T as the B operand (k = key, n = head): transpose the two
            // 8x8 halves of the S^T accumulator fragment
            const uint32_t pb0 = movmatrix_t(pack_bf16x2(p0, p1));
            const uint32_t pb1 = movmatrix_t(pack_bf16x2(p2, p3));
            // ---- O^T (d x heads) += V^T P^T over the warp's 16 keys
#pragma unroll
            for (int mt = 0; mt < D / 16; mt++) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(vaddr + sw128_offset(vrow_a, 2 * mt + vchunk_a), a0, a1, a2, a3);
                mma_bf16_16816(oacc[mt], a0, a1, a2, a3, pb0, pb1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        // row sums over the warp's keys: lanes with equal lane%4 hold the same heads
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
            l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
        }
    }
    __syncthreads();
    if (abort_flag && threadIdx.x == NC * 32) {
        // a wait gave up: let the copies still in flight land before the
        // ring is reused (bounded, no abort short-cut)
        const int issued = issued_sh;
        for (int i = max(0, issued - NS); i < issued; i++)
            mbar_wait(&full[i % NS], (i / NS) & 1, nullptr, 43, 100000000ull);
    }
    __syncthreads();

    // ---- warp partials (m, l, O) into the idle ring
    if (warp < NC) {
        float *wp = part + warp * PF;
        const int hn = lane >> 2, qc = (lane & 3) * 2;
        if (lane < 4) {
            wp[qc] = m_run[0];
            wp[qc + 1] = m_run[1];
            wp[8 + qc] = l_run[0];
            wp[8 + qc + 1] = l_run[1];
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; mt++) {
            wp[16 + qc * D + 16 * mt + hn] = oacc[mt][0];
            wp[16 + (qc + 1) * D + 16 * mt + hn] = oacc[mt][1];
            wp[16 + qc * D + 16 * mt + 8 + hn] = oacc[mt][2];
            wp[16 + (qc + 1) * D + 16 * mt + 8 + hn] = oacc[mt][3];
        }
    }
    // ---- one merge over the row's P x NC partials (distributed shared memory)
    cluster.sync();
    const int nsrc = P * NC;
    for (int e = threadIdx.x; e < nsrc * G; e += C::THREADS) {
        const int src = e / G, h = e % G;
        const float *pp = cluster.map_shared_rank(part, src / NC) + (src % NC) * PF;
        wgt[src][h] = pp[h];          // m, turned into a weight below
        lsrc[src][h] = pp[8 + h];
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float mc = -INFINITY;
        for (int src = 0; src < nsrc; src++) mc = fmaxf(mc, wgt[src][h]);
        float lc = 0.f;
        for (int src = 0; src < nsrc; src++) {
            const float f = mc == -INFINITY ? 0.f : fast_exp2(wgt[src][h] - mc);
            wgt[src][h] = f;
            lc += f * lsrc[src][h];
        }
        inv_l[h] = lc > 0.f ? 1.f / lc : 0.f;
    }
    __syncthreads();
    {
        const int n4 = G * D / 4;
        const int per = (n4 + P - 1) / P;
        const int e_end = min(n4, (rank + 1) * per);
        for (int e4 = rank * per + threadIdx.x; e4 < e_end; e4 += C::THREADS) {
            const int h = (e4 * 4) / D, c = (e4 * 4) % D;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int src = 0; src < nsrc; src++) {
                const float f = wgt[src][h];
                const float4 x = *reinterpret_cast<const float4 *>(
                    cluster.map_shared_rank(part, src / NC) + (src % NC) * PF + 16 + h * D + c);
                acc.x += f * x.x;
                acc.y += f * x.y;
                acc.z += f * x.z;
                acc.w += f * x.w;
            }
            const float il = inv_l[h];
            uint2 out;
            out.x = pack_bf16x2(acc.x * il, acc.y * il);
            out.y = pack_bf16x2(acc.z * il, acc.w * il);
            *reinterpret_cast<uint2 *>(o + ((long)b * Hq + g * G + h) * D + c) = out;
        }
    }
    cluster.sync();   // the other CTAs' shared memory must outlive the reads into it
}

}  // namespace qsa
