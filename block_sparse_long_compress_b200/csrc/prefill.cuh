// Step 5 (prefill) -- exact softmax attention over the selected blocks only
// (page "Qwen4 architecture: QSA, GR, PLE", section 1, "attend closely to
// the selected regions"; page "Qwen4 in llama.cpp: Dissecting PR #27742",
// section "QSA Is an Address-Selection Problem, Not a New Attention
// Equation": ordinary attention over the visible cells).
//
// Work unit (one CTA): 128 MMA rows = TOK query tokens x G query heads of
// one KV group (row r = token (r / G), head (r % G)), all sharing the same
// selected key blocks.  Per selected block n:
//     S = Q K_n^T          tcgen05.mma kind::f16, A = Q (smem, K-major),
//                          B = K block (smem, K-major), D = S (TMEM, fp32)
//     P = exp2(S*c - m)    softmax warps: tcgen05.ld S, online max/sum,
//                          write P as bf16 back over S in TMEM
//     O += P V_n           tcgen05.mma, A = P (TMEM), B = V block (smem,
//                          MN-major), D = O (TMEM, fp32)
// K/V blocks arrive by TMA (128-byte swizzle, 64 x 64 element boxes) into a
// two-stage ring.  S is double-buffered in TMEM so that the softmax of block
// n overlaps the QK^T of block n+1.  The running max is only moved (and O
// rescaled in TMEM) when a block's max exceeds it by more than 2^8, so
// rescales are rare.
//
// Warp roles (192 threads): warps 0-3 softmax + epilogue (thread = row =
// TMEM lane), warp 4 TMA producer, warp 5 TMEM allocator + MMA issuer.
// TMEM columns: O [0, D), S/P buffer b at [128 + 64 b, 192 + 64 b).
// Every mbarrier wait is bounded (QSA_ERR_TIMEOUT + early exit).
#pragma once
#include "device.cuh"

namespace qsa {

template <int D, int G>
struct PrefillCfg {
    static constexpr int M = 128;
    static constexpr int TOK = M / G;
    static constexpr int TILES = 64 / TOK;          // CTAs per 64-token query block
    static constexpr int NH = D / 64;               // 128-byte column halves
    static constexpr int Q_BYTES = M * D * 2;
    static constexpr int HALF_BYTES = 64 * 128;     // one 64x64 bf16 TMA box
    static constexpr int KV_BYTES = 64 * D * 2;     // one K (or V) block
    static constexpr int NS = 2;                    // K/V stages
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int SMEM_DATA = Q_BYTES + NS * STAGE_BYTES;
    static constexpr int THREADS = 192;
    static constexpr int TMEM_COLS = 256;
    static constexpr int S_COL = 128;
    // keep at most two CTAs per SM so their TMEM (2 x 256 columns) fits
    static constexpr int SMEM_REQUEST = (SMEM_DATA + 1024 > 80 * 1024) ? SMEM_DATA + 1024 : 80 * 1024;
};

struct PrefillShared {
    uint64_t q_full;
    uint64_t kv_full[2];
    uint64_t kv_empty[2];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint32_t tmem_base;
    int nblk;
    int abort;
    int blocks[64];
};

template <int D, int G>
__global__ void __launch_bounds__(192, 1) sparse_attn_prefill_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ idx,
    __nv_bfloat16 *__restrict__ O, float *__restrict__ lse, int Tq, int Hq, int Hkv,
    int q_pos0, int T_kv_max, int topk, float sm_scale_log2)
{
    using C = PrefillCfg<D, G>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ PrefillShared sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *q_smem = smem;
    uint8_t *kv_smem = smem + C::Q_BYTES;

    const int NR = (Tq + 63) / 64;
    const int i = blockIdx.x / C::TILES, sub = blockIdx.x % C::TILES;
    const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int token0 = i * 64 + sub * C::TOK;
    if (token0 >= Tq) return;   // ragged tail: whole CTA idle (uniform exit)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_last = min(i * 64 + 63, Tq - 1);
    const int Dg = (q_pos0 + row_last) / 64;

    if (threadIdx.x == 0) {
        // selected blocks of this row; stop at the first -1 or bad index
        const int32_t *sel = idx + ((long)bg * NR + i) * topk;
        int n = 0;
        for (int s = 0; s < topk; s++) {
            const int j = sel[s];
            if (j < 0) break;
            if (j > Dg || (n > 0 && j <= sh.blocks[n - 1])) {
                report(QSA_ERR_BOUNDS, 1);
                break;
            }
            sh.blocks[n++] = j;
        }
        if (n == 0) report(QSA_ERR_BOUNDS, 2);
        sh.nblk = n;
        sh.abort = 0;
        mbar_init(&sh.q_full, 1);
        for (int s = 0; s < 2; s++) {
            mbar_init(&sh.kv_full[s], 1);
            mbar_init(&sh.kv_empty[s], 1);
            mbar_init(&sh.s_full[s], 1);
            mbar_init(&sh.p_full[s], 128);
            mbar_init(&sh.pv_done[s], 1);
        }
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(&sh.tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int nblk = sh.nblk;
    volatile int *abort = &sh.abort;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && nblk > 0) {
            mbar_arrive_expect_tx(&sh.q_full, C::Q_BYTES);
            for (int h = 0; h < C::NH; h++)
                tma_load_3d(q_smem + h * (C::M * 128), &tmQ, &sh.q_full, h * 64, g * G,
                            b * Tq + token0);
            const long kv_row0 = (long)bg * T_kv_max;
            for (int n = 0; n < nblk; n++) {
                const int st = n % C::NS;
                if (n >= C::NS && !mbar_wait(&sh.kv_empty[st], ((n / C::NS) - 1) & 1, abort, 10))
                    break;
                uint8_t *ks = kv_smem + st * C::STAGE_BYTES;
                uint8_t *vs = ks + C::KV_BYTES;
                const int y = (int)(kv_row0 + 64L * sh.blocks[n]);
                mbar_arrive_expect_tx(&sh.kv_full[st], C::STAGE_BYTES);
                for (int h = 0; h < C::NH; h++) {
                    tma_load_2d(ks + h * C::HALF_BYTES, &tmK, &sh.kv_full[st], h * 64, y);
                    tma_load_2d(vs + h * C::HALF_BYTES, &tmV, &sh.kv_full[st], h * 64, y);
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------- MMA issuer
        if (lane == 0 && nblk > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc_bf16(128, D, 0, 1);
            bool ok = mbar_wait(&sh.q_full, 0, abort, 20);
            const uint32_t q_addr = smem_u32(q_smem);
            const uint32_t kv_addr = smem_u32(kv_smem);
            auto issue_s = [&](int n) -> bool {
                const int st = n % C::NS, buf = n & 1;
                if (!mbar_wait(&sh.kv_full[st], (n / C::NS) & 1, abort, 21)) return false;
                tc_fence_after();
                const uint32_t ks = kv_addr + st * C::STAGE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const uint32_t off = (kk & 3) * 32;   // 16 bf16 = 32 B inside a 128 B swizzle row
                    const uint64_t ad = umma_smem_desc(q_addr + (kk >> 2) * (C::M * 128) + off, 16, 1024);
                    const uint64_t bd = umma_smem_desc(ks + (kk >> 2) * C::HALF_BYTES + off, 16, 1024);
                    umma_ss(tmem + C::S_COL + 64 * buf, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sh.s_full[buf]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int n = 0; ok && n < nblk; n++) {
                const int st = n % C::NS, buf = n & 1;
                if (n + 1 < nblk) {
                    // S buffer (n+1)&1 holds P(n-1) until PV(n-1) is done
                    if (n >= 1 && !mbar_wait(&sh.pv_done[(n + 1) & 1], ((n - 1) >> 1) & 1, abort, 22)) break;
                    if (!issue_s(n + 1)) break;
                }
                if (!mbar_wait(&sh.p_full[buf], (n >> 1) & 1, abort, 23)) break;
                tc_fence_after();
                const uint32_t vs = kv_addr + st * C::STAGE_BYTES + C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    const uint64_t bd = umma_smem_desc(vs + kk * 2048, C::HALF_BYTES, 1024);
                    umma_ts(tmem, tmem + C::S_COL + 64 * buf + kk * 8, bd, idesc_o,
                            (n > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&sh.kv_empty[st]);
                umma_commit(&sh.pv_done[buf]);
            }
        }
    } else {
        // ------------------------------------------ softmax + epilogue
        const int r = threadIdx.x;                       // row = TMEM lane
        const int tok = token0 + r / G;
        const long p = (long)q_pos0 + tok;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        float m_run = -INFINITY, l = 0.f;
        bool ok = nblk > 0;
        for (int n = 0; ok && n < nblk; n++) {
            const int buf = n & 1;
            if (!mbar_wait(&sh.s_full[buf], (n >> 1) & 1, abort, 30)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[64];
            tmem_ld32(lane_addr + C::S_COL + 64 * buf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(lane_addr + C::S_COL + 64 * buf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
            float s[64];
#pragma unroll
            for (int c = 0; c < 64; c++) s[c] = __uint_as_float(sr[c]);
            if (sh.blocks[n] == Dg) {
                // only the diagonal block has keys after some rows' positions
                const long limit = p - 64L * Dg;
#pragma unroll
                for (int c = 0; c < 64; c++)
                    if (c > limit) s[c] = -INFINITY;
            }
            float q0 = s[0], q1 = s[16], q2 = s[32], q3 = s[48];
#pragma unroll
            for (int c = 1; c < 15; c += 2) {
                q0 = max3f(q0, s[c], s[c + 1]);
                q1 = max3f(q1, s[16 + c], s[17 + c]);
                q2 = max3f(q2, s[32 + c], s[33 + c]);
                q3 = max3f(q3, s[48 + c], s[49 + c]);
            }
            const float mx = max3f(max3f(q0, q1, s[15]), max3f(q2, q3, s[31]), fmaxf(s[47], s[63])) *
                             sm_scale_log2;
            if (n == 0) {
                m_run = mx;
            } else if (__any_sync(0xffffffffu, mx > m_run + 8.0f)) {
                const float m_new = fmaxf(m_run, mx);
                const float alpha = fast_exp2(m_run - m_new);
                // O is stable once PV(n-1) has completed
                if (!mbar_wait(&sh.pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort, 31)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_addr + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; c++) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st32(lane_addr + c0, o);
                }
                tmem_wait_st();
                l *= alpha;
                m_run = m_new;
            }
            // P = 2^(s*c - m): 3 of every 8 pairs on the FMA pipe, the rest on MUFU
            uint32_t pk[32];
            const uint64_t sc2 = f2_pack(sm_scale_log2, sm_scale_log2);
            const uint64_t nm2 = f2_pack(-m_run, -m_run);
            uint64_t lacc = f2_pack(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 32; c++) {
                const uint64_t x2 = f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), sc2, nm2);
                uint64_t p2;
                if ((c & 7) == 1 || (c & 7) == 4 || (c & 7) == 6) {
                    p2 = exp2_poly_x2(x2);
                } else {
                    float x0, x1;
                    f2_unpack(x2, x0, x1);
                    p2 = f2_pack(fast_exp2(x0), fast_exp2(x1));
                }
                lacc = f2_add(lacc, p2);
                float p0, p1;
                f2_unpack(p2, p0, p1);
                pk[c] = pack_bf16x2(p0, p1);
            }
            float la, lb;
            f2_unpack(lacc, la, lb);
            const float lsum = la + lb;
            l += lsum;
            tmem_st32(lane_addr + C::S_COL + 64 * buf, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sh.p_full[buf]);
        }
        if (ok && !mbar_wait(&sh.pv_done[(nblk - 1) & 1], ((nblk - 1) >> 1) & 1, abort, 32)) ok = false;
        tc_fence_after();
        const bool store = tok < Tq;
        const int h = g * G + r % G;
        __nv_bfloat16 *orow = O + (((long)b * Tq + tok) * Hq + h) * D;
        const float inv_l = (ok && l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(lane_addr + c0, o);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; c++)
                pk[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
            if (store) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                for (int v = 0; v < 4; v++)
                    dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
        }
        if (store && lse)
            lse[((long)b * Tq + tok) * Hq + h] =
                (ok && l > 0.f) ? (m_run + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace qsa
