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
// The row's partials merge through distributed shared memory: each CTA
// combines its 4 warps' (max, sum, O) per head, then pushes the result into
// the inbox of the CTA that finishes that head (head h -> CTA h mod P) with
// plain remote stores between two cluster barriers; each owner merges its
// inbox locally.  No global workspace, no global atomics, no remote loads.
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

// FP8: the rotated fp8 cache option (quant.cuh): a stage holds two blocks'
// K and V codes (one 64 x 128-byte box each) and per-row scales; every
// consumer thread loads the codes of its MMA fragments straight from the
// stage and expands them to f16 in registers.
template <int D, bool FP8 = false>
struct DecodeCfg {
    static constexpr int NH = D / 64;                  // 64-column TMA boxes per row
    static constexpr int HALF_BYTES = 64 * 128;        // one 64-row x 128-byte box
    static constexpr int KV_BYTES = FP8 ? 64 * D : 64 * D * 2;   // one block's K (or V)
    static constexpr int SCALE_BYTES = FP8 ? 64 * 4 : 0;         // its per-row scales
    // FP8: a stage holds two blocks (codes and scales of each, 1024-aligned),
    // so that one full/empty round trip moves as many bytes as a bf16 block
    static constexpr int BLK_BYTES = FP8 ? (2 * KV_BYTES + 2 * SCALE_BYTES + 1023) / 1024 * 1024 : 2 * KV_BYTES;
    static constexpr int BPS = FP8 ? 2 : 1;            // blocks per stage
    static constexpr int STAGE_BYTES = BPS * BLK_BYTES;
    static constexpr int CTAS_PER_SM = 2;
    static constexpr int RING_BYTES = FP8 ? 3 * STAGE_BYTES : 96 * 1024;   // NS stages; two CTAs per SM
    static constexpr int NS = RING_BYTES / STAGE_BYTES;
    static constexpr int NC = 4;                       // consumer warps
    static constexpr int THREADS = (NC + 1) * 32;
    static constexpr int PART_FLOATS = 16 + 8 * D;     // m[8], l[8], O[8][D] of one warp
    static constexpr int SMEM_BYTES = RING_BYTES + 1024;
    static constexpr int MAX_SLOTS = 64;
    static constexpr int MAX_CLUSTER = 8;
    static_assert(NS >= 2, "ring too small");
    static_assert(NC * PART_FLOATS * 4 + 4 * D <= RING_BYTES, "merge scratch must fit in the ring");
    static_assert(!FP8 || D == 128, "rotated fp8 rows are 128 wide");
    // the merge inbox follows the ring in dynamic shared memory: ceil(G/P) * P
    // slots of (max, sum, 2 pad, O[D]) floats, sized by the host for its P
    static constexpr int SLOT_FLOATS = 4 + D;
    __host__ __device__ static constexpr int inbox_bytes(int G, int P) { return (G + P - 1) / P * P * SLOT_FLOATS * 4; }
};

__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Two e4m3 codes (low and high byte of a 16-bit half of w) to f16x2.
__device__ __forceinline__ uint32_t e4m3_lo(uint32_t w) { return cvt_e4m3x2_f16x2((uint16_t)(w & 0xFFFFu)); }
__device__ __forceinline__ uint32_t e4m3_hi(uint32_t w) { return cvt_e4m3x2_f16x2((uint16_t)(w >> 16)); }

__device__ __forceinline__ uint32_t u4_word(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

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

template <int D, int G, bool FP8 = false>
__global__ void __launch_bounds__(DecodeCfg<D, FP8>::THREADS, DecodeCfg<D, FP8>::CTAS_PER_SM) decode_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ idx,
    __nv_bfloat16 *__restrict__ o, int Hq, int Hkv, int L, int T_kv_max, int topk, int spc,
    float sm_scale_log2, const int32_t *__restrict__ seq_lens, const int32_t *__restrict__ block_table,
    int max_blocks, int num_pages, const float *__restrict__ k_scales, const float *__restrict__ v_scales)
{
    using C = DecodeCfg<D, FP8>;
    constexpr int NS = C::NS;
    constexpr int NC = C::NC;
    constexpr int PF = C::PART_FLOATS;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full[NS], empty[NS];
    __shared__ int blocks[C::MAX_SLOTS];   // the CTA's valid block ids in slot order
    __shared__ int rows[C::MAX_SLOTS];     // and the first cache row of each (TMA coordinate)
    __shared__ int nb_sh, issued_sh, abort_flag;
    __shared__ int ring_bad;               // a copy may still land in the ring (see the drain)
    __shared__ float wloc[NC][8];          // merge weights of the CTA's warps, per head
    __shared__ float mloc[8], lloc[8];     // the CTA's combined max and sum per head
    __shared__ __align__(16) uint32_t uq[FP8 ? 8 * (D / 2) : 1];   // FP8: rotated queries, f16 pairs

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
    // the group's queries, loaded by the consumer warps first thing, ahead
    // of the cache copies that every CTA starts after the prologue.  B
    // operand of S^T = K q^T: column n = head lane/4 of the group (zero for
    // n >= G), rows k = d; FP8: raw rows of heads warp, warp + NC, ...,
    // rotated below
    const int hn = lane >> 2, qc = (lane & 3) * 2;
    uint32_t qb[D / 16][2];
    uint2 qraw[FP8 ? (G + NC - 1) / NC : 1];
    if (warp < NC) {
        if constexpr (FP8) {
#pragma unroll
            for (int j = 0; j < (G + NC - 1) / NC; j++)
                if (warp + j * NC < G)
                    qraw[j] = __ldg(reinterpret_cast<const uint2 *>(q + ((long)b * Hq + g * G + warp + j * NC) * D) + lane);
        } else {
            const __nv_bfloat16 *qrow = q + ((long)b * Hq + g * G + (hn < G ? hn : 0)) * D;
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                const uint32_t lo = __ldg(reinterpret_cast<const uint32_t *>(qrow + 16 * kk + qc));
                const uint32_t hi = __ldg(reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 8 + qc));
                qb[kk][0] = hn < G ? lo : 0u;
                qb[kk][1] = hn < G ? hi : 0u;
            }
        }
    }
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
        ring_bad = 0;
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
            // slot i holds blocks BPS*i .. BPS*i + BPS - 1 (fewer at the end)
            const int nslots = (nb + C::BPS - 1) / C::BPS;
            int i = 0;
            for (; i < nslots; i++) {
                const int st = i % NS;
                if (i >= NS) {
                    if (!mbar_wait(&empty[st], ((i / NS) - 1) & 1, &abort_flag, 42)) break;
                    fence_proxy_async_smem();
                }
                uint8_t *ks = ring + st * C::STAGE_BYTES;
                uint8_t *vs = ks + C::KV_BYTES;
                if constexpr (FP8) {
                    // per block: codes, one 64-row x 128-byte box each; scales,
                    // 64 fp32 per tensor, one plain bulk copy each
                    const int nbk = min(C::BPS, nb - C::BPS * i);
                    mbar_arrive_expect_tx(&full[st], nbk * (2 * C::KV_BYTES + 2 * C::SCALE_BYTES));
                    for (int h = 0; h < nbk; h++) {
                        const int row = rows[C::BPS * i + h];
                        uint8_t *kb = ks + h * C::BLK_BYTES;
                        uint8_t *vb = kb + C::KV_BYTES;
                        tma_load_2d(kb, &tmK, &full[st], 0, row);
                        tma_load_2d(vb, &tmV, &full[st], 0, row);
                        bulk_load(vb + C::KV_BYTES, k_scales + row, C::SCALE_BYTES, &full[st]);
                        bulk_load(vb + C::KV_BYTES + C::SCALE_BYTES, v_scales + row, C::SCALE_BYTES, &full[st]);
                    }
                } else {
                    const int row = rows[i];
                    mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
#pragma unroll
                    for (int h = 0; h < C::NH; h++)
                        tma_load_2d(ks + h * C::HALF_BYTES, &tmK, &full[st], h * 64, row);
#pragma unroll
                    for (int h = 0; h < C::NH; h++)
                        tma_load_2d(vs + h * C::HALF_BYTES, &tmV, &full[st], h * 64, row);
                }
            }
            issued_sh = i;
        }
    } else {
        // ---------------------------------------------------- consumers
        if constexpr (FP8) {
            // the group's queries in the rotated basis (unnormalised
            // transform, as f16 pairs), shared among the consumer warps only
#pragma unroll
            for (int j = 0; j < (G + NC - 1) / NC; j++) {
                const int h = warp + j * NC;
                if (h < G) {
                    const uint2 raw = qraw[j];
                    float x[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                                  __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
                    fwht_warp<4>(x);
                    uq[h * (D / 2) + 2 * lane] = pack_f16x2(x[0], x[1]);
                    uq[h * (D / 2) + 2 * lane + 1] = pack_f16x2(x[2], x[3]);
                }
            }
            named_barrier_sync(1, NC * 32);
            // rotated queries (f16) from the shared copy.  The contraction
            // over d runs in a permuted order that gives every thread 32
            // contiguous codes of each of its key rows: in k-step kk, MMA k
            // indices 2c, 2c + 1 (c = lane % 4) stand for d = 32c + 4kk + {0, 1}
            // and 2c + 8, 2c + 9 for d = 32c + 4kk + {2, 3}.
            const uint32_t *uqh = uq + (hn < G ? hn : 0) * (D / 2);
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                qb[kk][0] = hn < G ? uqh[8 * qc + 2 * kk] : 0u;
                qb[kk][1] = hn < G ? uqh[8 * qc + 2 * kk + 1] : 0u;
            }
        }
        const int k0 = 16 * warp;                                  // the warp's keys in each block
        const int krow_a = k0 + (lane & 7) + 8 * ((lane >> 3) & 1);  // K rows for ldmatrix (A of S^T)
        const int kchunk_a = lane >> 4;
        const int vrow_a = k0 + (lane & 7) + 8 * (lane >> 4);        // V rows for ldmatrix.trans (A of O^T)
        const int vchunk_a = (lane >> 3) & 1;
        const int key_lo = k0 + (lane >> 2);                         // keys of this thread's S^T entries
        if constexpr (FP8) {
            // Two blocks per iteration (one softmax update for both): the
            // per-block chain (codes -> S MMAs -> row max -> exponentials ->
            // PV MMAs) is latency-bound with two consumer warps per
            // scheduler, and the pair doubles the independent work in it.
            const int c = lane & 3, r = lane >> 2, sw = key_lo & 7;   // (key_lo + 8) & 7 == sw
            const float sc = sm_scale_log2 * (1.0f / 128.0f);
            // the thread's codes, straight from the stage (128-byte swizzle):
            // K rows key_lo and key_lo + 8, bytes 32c .. 32c+31; V rows
            // k0 + {2c, 2c+1, 2c+8, 2c+9}, bytes 16r .. 16r+15; and the
            // per-row scales (scores: (u_q . u_k) / 128 = q . k with
            // u_k = scale * code; the V scale rides on P)
            auto load = [&](const uint8_t *kst, uint4 (&kr)[4], uint4 (&vr)[4], float (&kq)[2], float (&vp)[2]) {
                const uint8_t *vst = kst + C::KV_BYTES;
                const float *ksc = reinterpret_cast<const float *>(vst + C::KV_BYTES);
                const float *vsc = ksc + 64;
                kr[0] = *reinterpret_cast<const uint4 *>(kst + key_lo * 128 + (((2 * c) ^ sw) << 4));
                kr[1] = *reinterpret_cast<const uint4 *>(kst + key_lo * 128 + (((2 * c + 1) ^ sw) << 4));
                kr[2] = *reinterpret_cast<const uint4 *>(kst + (key_lo + 8) * 128 + (((2 * c) ^ sw) << 4));
                kr[3] = *reinterpret_cast<const uint4 *>(kst + (key_lo + 8) * 128 + (((2 * c + 1) ^ sw) << 4));
#pragma unroll
                for (int t = 0; t < 4; t++) {
                    const int vk = k0 + 2 * c + (t & 1) + 8 * (t >> 1);
                    vr[t] = *reinterpret_cast<const uint4 *>(vst + vk * 128 + ((r ^ (vk & 7)) << 4));
                }
                kq[0] = ksc[key_lo] * sc;
                kq[1] = ksc[key_lo + 8] * sc;
                vp[0] = vsc[key_lo];
                vp[1] = vsc[key_lo + 8];
            };
            // S^T (16 keys x 8 heads) = K q^T, two independent chains
            auto scores = [&](const uint4 (&kr)[4], float (&s)[4]) {
                float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const uint32_t wl = u4_word(kr[kk >> 2], kk & 3);        // row key_lo
                    const uint32_t wh = u4_word(kr[2 + (kk >> 2)], kk & 3);  // row key_lo + 8
                    if (kk & 1)
                        mma_f16_16816(s2, e4m3_lo(wl), e4m3_lo(wh), e4m3_hi(wl), e4m3_hi(wh), qb[kk][0], qb[kk][1]);
                    else
                        mma_f16_16816(s, e4m3_lo(wl), e4m3_lo(wh), e4m3_hi(wl), e4m3_hi(wh), qb[kk][0], qb[kk][1]);
                }
#pragma unroll
                for (int t = 0; t < 4; t++) s[t] += s2[t];
            };
            // keys c <= lim of the block are visible; scaled scores or -inf
            auto mask_scale = [&](float (&s)[4], int lim, const float (&kq)[2]) {
                const bool v0 = key_lo <= lim, v1 = key_lo + 8 <= lim;
                s[0] = v0 ? s[0] * kq[0] : -INFINITY;
                s[1] = v0 ? s[1] * kq[0] : -INFINITY;
                s[2] = v1 ? s[2] * kq[1] : -INFINITY;
                s[3] = v1 ? s[3] * kq[1] : -INFINITY;
            };
            // O^T += V^T P^T: MMA rows (mt, r) and (mt, r + 8) stand for
            // d = 16r + 2mt and 16r + 2mt + 1, i.e. bytes 2mt, 2mt + 1 of the
            // thread's chunk of each key, paired across keys by a byte permute
            auto pv = [&](const uint4 (&vr)[4], uint32_t pb0, uint32_t pb1) {
#pragma unroll
                for (int mt = 0; mt < D / 16; mt++) {
                    const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
                    const uint32_t pa = prmt(u4_word(vr[0], mt >> 1), u4_word(vr[1], mt >> 1), sel);
                    const uint32_t pc = prmt(u4_word(vr[2], mt >> 1), u4_word(vr[3], mt >> 1), sel);
                    mma_f16_16816(oacc[mt], e4m3_lo(pa), e4m3_hi(pa), e4m3_lo(pc), e4m3_hi(pc), pb0, pb1);
                }
            };
            static_assert(!FP8 || C::BPS == 2, "a stage holds the pair");
            for (int i = 0; i < nb; i += 2) {
                const bool two = i + 1 < nb;   // warp-uniform
                const int slot = i / 2, st = slot % NS;
                if (!mbar_wait(&full[st], (slot / NS) & 1, &abort_flag, 40)) break;
                const uint8_t *stage = ring + st * C::STAGE_BYTES;
                uint4 kra[4], vra[4], krb[4], vrb[4];
                float kqa[2], vpa[2], kqb[2] = {0.f, 0.f}, vpb[2] = {0.f, 0.f};
                load(stage, kra, vra, kqa, vpa);
                if (two) load(stage + C::BLK_BYTES, krb, vrb, kqb, vpb);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                float xa[4] = {0.f, 0.f, 0.f, 0.f}, xb[4] = {0.f, 0.f, 0.f, 0.f};
                scores(kra, xa);
                if (two) scores(krb, xb);
                mask_scale(xa, (Lb - 1) - 64 * blocks[i], kqa);
                mask_scale(xb, two ? (Lb - 1) - 64 * blocks[i + 1] : -1, kqb);
                // ---- online softmax per head over the warp's keys of both blocks
                float mx0 = fmaxf(fmaxf(xa[0], xa[2]), fmaxf(xb[0], xb[2]));
                float mx1 = fmaxf(fmaxf(xa[1], xa[3]), fmaxf(xb[1], xb[3]));
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
                const float pa0 = fast_exp2(xa[0] - mu0), pa1 = fast_exp2(xa[1] - mu1);
                const float pa2 = fast_exp2(xa[2] - mu0), pa3 = fast_exp2(xa[3] - mu1);
                const float pb0 = fast_exp2(xb[0] - mu0), pb1 = fast_exp2(xb[1] - mu1);
                const float pb2 = fast_exp2(xb[2] - mu0), pb3 = fast_exp2(xb[3] - mu1);
                l_run[0] = l_run[0] * al0 + ((pa0 + pa2) + (pb0 + pb2));
                l_run[1] = l_run[1] * al1 + ((pa1 + pa3) + (pb1 + pb3));
#pragma unroll
                for (int mt = 0; mt < D / 16; mt++) {
                    oacc[mt][0] *= al0;
                    oacc[mt][1] *= al1;
                    oacc[mt][2] *= al0;
                    oacc[mt][3] *= al1;
                }
                // P^T as the B operand (k = key, n = head): transpose the two
                // 8x8 halves of the S^T accumulator fragment
                pv(vra, movmatrix_t(pack_f16x2(pa0 * vpa[0], pa1 * vpa[0])),
                   movmatrix_t(pack_f16x2(pa2 * vpa[1], pa3 * vpa[1])));
                if (two)
                    pv(vrb, movmatrix_t(pack_f16x2(pb0 * vpb[0], pb1 * vpb[0])),
                       movmatrix_t(pack_f16x2(pb2 * vpb[1], pb3 * vpb[1])));
            }
        } else {
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
        // ring is reused (bounded, no abort short-cut).  If one still has
        // not landed, the ring is not reused at all: this CTA contributes
        // nothing to the merge and writes zeros for the heads it owns (the
        // timeout is in the status word either way)
        const int issued = issued_sh;
        for (int i = max(0, issued - NS); i < issued; i++)
            if (!mbar_wait(&full[i % NS], (i / NS) & 1, nullptr, 43, 100000000ull)) ring_bad = 1;
    }
    __syncthreads();
    const bool ring_ok = ring_bad == 0;

    // ---- warp partials (m, l, O) into the idle ring
    if (warp < NC && ring_ok) {
        float *wp = part + warp * PF;
        if (lane < 4) {
            wp[qc] = m_run[0];
            wp[qc + 1] = m_run[1];
            wp[8 + qc] = l_run[0];
            wp[8 + qc + 1] = l_run[1];
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; mt++) {
            // MMA row (mt, i) of O^T is d = 16mt + i, or in the fp8 order
            // d = 16i + 2mt (i < 8) and 16(i - 8) + 2mt + 1
            const int d0 = FP8 ? 16 * hn + 2 * mt : 16 * mt + hn;
            const int d1 = FP8 ? 16 * hn + 2 * mt + 1 : 16 * mt + 8 + hn;
            wp[16 + qc * D + d0] = oacc[mt][0];
            wp[16 + (qc + 1) * D + d0] = oacc[mt][1];
            wp[16 + qc * D + d1] = oacc[mt][2];
            wp[16 + (qc + 1) * D + d1] = oacc[mt][3];
        }
    }
    __syncthreads();
    // ---- merge.  Head h of the group is finished by CTA h % P of the
    // cluster.  Each CTA combines its NC warps per head, then stores its
    // combined (max, sum, unnormalised O) into slot [h / P][its rank] of the
    // owner's inbox with plain stores through distributed shared memory --
    // at once, while slower CTAs may still be streaming: the inbox has
    // shared memory of its own (after the ring), which nothing else uses;
    // after one cluster barrier each owner merges its inbox locally.
    constexpr int SLOT = C::SLOT_FLOATS;                 // max, sum, 2 pad, O[D]
    float *inbox = reinterpret_cast<float *>(ring + C::RING_BYTES);   // [ceil(G/P)][P][SLOT]
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float mc = -INFINITY;
        if (ring_ok) {
#pragma unroll
            for (int w = 0; w < NC; w++) mc = fmaxf(mc, part[w * PF + h]);
        }
        float lc = 0.f;
#pragma unroll
        for (int w = 0; w < NC; w++) {
            const float f = mc == -INFINITY ? 0.f : fast_exp2(part[w * PF + h] - mc);
            wloc[w][h] = f;
            lc += f * (ring_ok ? part[w * PF + 8 + h] : 0.f);
        }
        mloc[h] = mc;
        lloc[h] = lc;
    }
    __syncthreads();   // the local weights are visible
    for (int e4 = threadIdx.x; e4 < G * D / 4; e4 += C::THREADS) {
        const int h = (e4 * 4) / D, c = (e4 * 4) % D;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NC && ring_ok; w++) {
            const float f = wloc[w][h];
            const float4 x = *reinterpret_cast<const float4 *>(part + w * PF + 16 + h * D + c);
            acc.x += f * x.x;
            acc.y += f * x.y;
            acc.z += f * x.z;
            acc.w += f * x.w;
        }
        float *slot = cluster.map_shared_rank(inbox, h % P) + ((h / P) * P + rank) * SLOT;
        *reinterpret_cast<float4 *>(slot + 4 + c) = acc;
    }
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float *slot = cluster.map_shared_rank(inbox, h % P) + ((h / P) * P + rank) * SLOT;
        slot[0] = mloc[h];
        slot[1] = lloc[h];
    }
    cluster.sync();   // the inboxes are complete; no shared memory is read remotely after this
    // one warp per owned head: lane owns D/32 consecutive columns
    constexpr int CPL = D / 32;
    for (int j = warp; j * P + rank < G; j += NC + 1) {
        const int h = j * P + rank;
        const float *sl = inbox + j * P * SLOT;
        float mc = -INFINITY;
        for (int src = 0; src < P; src++) mc = fmaxf(mc, sl[src * SLOT]);
        float lc = 0.f, x[CPL];
#pragma unroll
        for (int t = 0; t < CPL; t++) x[t] = 0.f;
        for (int src = 0; src < P && ring_ok; src++) {
            const float f = mc == -INFINITY ? 0.f : fast_exp2(sl[src * SLOT] - mc);
            lc += f * sl[src * SLOT + 1];
#pragma unroll
            for (int t = 0; t < CPL; t++) x[t] += f * sl[src * SLOT + 4 + CPL * lane + t];
        }
        float il = lc > 0.f && ring_ok ? 1.f / lc : 0.f;
        if constexpr (FP8) {
            // back to the original basis: o = WHT(o') / 128 (the transform
            // squared is 128 I)
            fwht_warp<CPL>(x);
            il *= 1.0f / 128.0f;
        }
        __nv_bfloat16 *orow = o + ((long)b * Hq + g * G + h) * D + CPL * lane;
        if constexpr (CPL == 4) {
            uint2 out;
            out.x = pack_bf16x2(x[0] * il, x[1] * il);
            out.y = pack_bf16x2(x[2] * il, x[3] * il);
            *reinterpret_cast<uint2 *>(orow) = out;
        } else {
            *reinterpret_cast<uint32_t *>(orow) = pack_bf16x2(x[0] * il, x[1] * il);
        }
    }
}

}  // namespace qsa
