// Step 5 (prefill) -- exact softmax attention over the selected blocks only
// (page "Qwen4 architecture: QSA, GR, PLE", section 1, "attend closely to
// the selected regions"; page "Qwen4 in llama.cpp: Dissecting PR #27742",
// section "QSA Is an Address-Selection Problem, Not a New Attention
// Equation": ordinary attention over the visible cells).
//
// Work unit (one CTA, one per SM): two 128-row MMA tiles of one KV group
// and query block; row r of a tile = token (r / G), query head (r % G) --
// 256 rows sharing the same selected key blocks, so every gathered K/V
// block is loaded once for all 256 rows.  Selected blocks are consumed in
// pairs (128 keys; an odd last pair repeats its first block and masks the
// copy) through separate 2-deep K and V rings: a K stage is released once
// both tiles' S are done, well before its V stage.  Per pair n and tile t:
//     S_t = Q_t K_n^T       tcgen05.mma kind::f16, M=128 N=128 K=16 steps,
//                           A = Q_t, B = the pair's keys (both K-major in
//                           shared memory), D = S_t in TMEM (fp32)
//     P_t = 2^(S_t c - m)   softmax warpgroup t, one thread per row holding
//                           all 128 scores in registers; bf16 P_t is written
//                           over the first 64 columns of S_t
//     O_t += P_t V_n        tcgen05.mma, A = P_t from TMEM, B = the pair's
//                           values (MN-major in shared memory), D = O_t
// Each tile has its own MMA-issuing thread, so while one waits for its
// softmax the other keeps the tensor pipe fed (an mbarrier query stalls the
// issuing thread for a few hundred cycles, longer than the MMA queue
// covers).  The two issuers hand the pipe back and forth through "S issued"
// barriers so that its work strictly alternates between the tiles:
//     S0(0) | S1(0) | PV0(0) S0(1) | PV1(0) S1(1) | PV0(1) S0(2) | ...
// and each tile's softmax runs while the pipe works on the other tile (left
// free, two identical chains drift into lockstep and their softmaxes then
// compete for the same issue slots while the pipe idles).  Within a tile, S_t(n+1) is issued after PV_t(n) by the same
// thread; the tensor pipe runs a thread's MMAs in order, so P_t(n) is read
// before S_t(n+1) overwrites it.  The running max only moves (and O_t is
// rescaled in TMEM) when a pair's max exceeds it by more than 2^8.
//
// Warps (384 threads, three warpgroups): 0-7 softmax/epilogue (tile =
// warp/4, TMEM lane quarter = warp%4, thread = row; a row's 128 scores stay
// in registers from the max to the exponentials), 8 TMA producer, 9 TMEM
// allocator + MMA issuer of tile 0, 10 MMA issuer of tile 1, 11 idle.  The
// last warpgroup gives registers to the softmax warpgroups (setmaxnreg).
// Each softmax warp signals P with a single arrive.
// TMEM (512 columns): O_0 [0,128) O_1 [128,256) S_0 [256,384) S_1 [384,512);
// P_t in S_t columns [0,64).  Every mbarrier wait is bounded.
#pragma once
#include "device.cuh"

namespace qsa {

template <int D, int G>
struct PrefillCfg {
    static constexpr int M = 128;                  // rows per tile
    static constexpr int TOK = M / G;              // tokens per tile
    static constexpr int TILES = 64 / (2 * TOK);   // CTAs per 64-token query block
    static constexpr int NH = D / 64;              // 128-byte column halves
    static constexpr int HALF_ROWS_BYTES = 128 * 128;   // 128 rows x 128 B (one half of a tile)
    static constexpr int QT_BYTES = NH * HALF_ROWS_BYTES;   // one Q tile
    static constexpr int PAIR_BYTES = NH * HALF_ROWS_BYTES; // K (or V) of a block pair
    static constexpr int NS = 2;                   // K stages and V stages (pairs)
    static constexpr int SMEM_DATA = 2 * QT_BYTES + 2 * NS * PAIR_BYTES;
    // the CTA owns all 512 TMEM columns: ask for enough shared memory that
    // a second CTA never lands on the same SM
    static constexpr int SMEM_REQUEST = (SMEM_DATA + 1024 > 120 * 1024) ? SMEM_DATA + 1024 : 120 * 1024;
    static constexpr int THREADS = 12 * 32;
    // registers: launched at REG_LAUNCH per thread (the launch bounds'
    // ceiling for 384 threads, checked by the build); the producer/issuer
    // warpgroup drops to REG_LOW and the two softmax warpgroups, which hold
    // a row's 128 scores, rise to REG_HIGH: 256 * REG_HIGH + 128 * REG_LOW
    // must not exceed 384 * REG_LAUNCH
    static constexpr int REG_LAUNCH = 168;
    static constexpr int REG_LOW = 48;
    static constexpr int REG_HIGH = 224;
    static_assert(256 * REG_HIGH + 128 * REG_LOW <= 384 * REG_LAUNCH, "register split exceeds the launch pool");
    static constexpr int TMEM_COLS = 512;
    static constexpr int O_COL = 0, S_COL = 256;
};

struct PrefillShared {
    uint64_t q_full;
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2];
    uint64_t s_issued[2];
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint32_t tmem_base;
    int nblk;
    int abort;
    int blocks[64];
};

template <int D, int G>
__global__ void __launch_bounds__(12 * 32, 1) sparse_attn_prefill_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ idx,
    __nv_bfloat16 *__restrict__ O, float *__restrict__ lse, int Tq, int Hq, int Hkv,
    int q_pos0, int T_kv_max, int topk, float sm_scale_log2)
{
    using C = PrefillCfg<D, G>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ PrefillShared sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *q_smem = smem;                          // [tile][half][128 rows][128 B]
    uint8_t *k_smem = smem + 2 * C::QT_BYTES;        // [stage][half][128 rows][128 B]
    uint8_t *v_smem = k_smem + C::NS * C::PAIR_BYTES;

    const int NR = (Tq + 63) / 64;
    const int i = blockIdx.x / C::TILES, sub = blockIdx.x % C::TILES;
    const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int token0 = i * 64 + sub * 2 * C::TOK;
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
        for (int s = 0; s < C::NS; s++) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 2);    // one arrive per tile
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 2);
        }
        for (int t = 0; t < 2; t++) {
            mbar_init(&sh.s_full[t], 1);
            mbar_init(&sh.s_issued[t], 1);
            mbar_init(&sh.p_full[t], 4);     // one arrive per softmax warp
            mbar_init(&sh.pv_done[t], 1);
        }
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(&sh.tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int nblk = sh.nblk;
    const int npair = (nblk + 1) / 2;
    volatile int *abort = &sh.abort;

    if (warp >= 8) {
    // warpgroup 2 (one setmaxnreg for its four warps): producer, issuers
    setmaxnreg_dec<C::REG_LOW>();
    if (warp == 8) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && nblk > 0) {
            mbar_arrive_expect_tx(&sh.q_full, 2 * C::QT_BYTES);
            for (int t = 0; t < 2; t++)
                for (int h = 0; h < C::NH; h++)
                    tma_load_3d(q_smem + t * C::QT_BYTES + h * C::HALF_ROWS_BYTES, &tmQ, &sh.q_full, h * 64,
                                g * G, b * Tq + token0 + t * C::TOK);
            const int kv_row0 = bg * T_kv_max;   // host checks B*Hkv*T_kv_max < 2^31
            for (int n = 0; n < npair; n++) {
                const int st = n % C::NS;
                const int ya = kv_row0 + 64 * sh.blocks[2 * n];
                // an odd last pair repeats its first block (its copy is masked)
                const int yb = kv_row0 + 64 * sh.blocks[2 * n + 1 < nblk ? 2 * n + 1 : 2 * n];
                if (n >= C::NS && !mbar_wait(&sh.k_empty[st], ((n / C::NS) - 1) & 1, abort, 10)) break;
                uint8_t *ks = k_smem + st * C::PAIR_BYTES;
                mbar_arrive_expect_tx(&sh.k_full[st], C::PAIR_BYTES);
                for (int h = 0; h < C::NH; h++) {
                    tma_load_2d(ks + h * C::HALF_ROWS_BYTES, &tmK, &sh.k_full[st], h * 64, ya);
                    tma_load_2d(ks + h * C::HALF_ROWS_BYTES + 64 * 128, &tmK, &sh.k_full[st], h * 64, yb);
                }
                if (n >= C::NS && !mbar_wait(&sh.v_empty[st], ((n / C::NS) - 1) & 1, abort, 11)) break;
                uint8_t *vs = v_smem + st * C::PAIR_BYTES;
                mbar_arrive_expect_tx(&sh.v_full[st], C::PAIR_BYTES);
                for (int h = 0; h < C::NH; h++) {
                    tma_load_2d(vs + h * C::HALF_ROWS_BYTES, &tmV, &sh.v_full[st], h * 64, ya);
                    tma_load_2d(vs + h * C::HALF_ROWS_BYTES + 64 * 128, &tmV, &sh.v_full[st], h * 64, yb);
                }
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ----------------------------------------- MMA issuer of tile t
        const int t = warp - 9;
        if (lane == 0 && nblk > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc_bf16(128, D, 0, 1);
            // descriptor bases, built once: per MMA only a 64-bit add of the
            // byte offset >> 4 into the start-address field remains (shared
            // memory addresses stay below 2^18, so the field never carries)
            const uint64_t qd = umma_smem_desc(smem_u32(q_smem + t * C::QT_BYTES), 16, 1024);
            const uint64_t kd = umma_smem_desc(smem_u32(k_smem), 16, 1024);
            const uint64_t vd = umma_smem_desc(smem_u32(v_smem), C::HALF_ROWS_BYTES, 1024);
            const uint32_t s_tmem = tmem + C::S_COL + 128 * t;
            const uint32_t o_tmem = tmem + C::O_COL + 128 * t;
            // S_t(n) = Q_t K(n)^T over the pair's 128 keys
            auto issue_s = [&](int n) {
                const uint64_t kds = kd + (uint64_t)(((n % C::NS) * C::PAIR_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const uint64_t off = (uint64_t)((((kk >> 2) * C::HALF_ROWS_BYTES) + (kk & 3) * 32) >> 4);
                    umma_ss(s_tmem, qd + off, kds + off, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sh.s_full[t]);
                mbar_arrive(&sh.s_issued[t]);
            };
            bool ok = mbar_wait(&sh.q_full, 0, abort, 20) && mbar_wait(&sh.k_full[0], 0, abort, 21);
            // tile 1's first S goes to the pipe right after tile 0's
            if (ok && t == 1) ok = mbar_wait(&sh.s_issued[0], 0, abort, 25);
            if (ok) {
                tc_fence_after();
                issue_s(0);
            }
            for (int n = 0; ok && n < npair; n++) {
                const int st = n % C::NS;
                const bool more = n + 1 < npair;
                // checks that are normally satisfied long ago, done while this
                // tile's S MMAs are still queued on the pipe
                if (!mbar_wait(&sh.v_full[st], (n / C::NS) & 1, abort, 26)) break;
                if (more && !mbar_wait(&sh.k_full[(n + 1) % C::NS], ((n + 1) / C::NS) & 1, abort, 21)) break;
                // alternate the pipe: PV0(n) after S1(n) was issued, PV1(n) after S0(n+1)
                if (t == 0 && !mbar_wait(&sh.s_issued[1], n & 1, abort, 27)) break;
                if (t == 1 && more && !mbar_wait(&sh.s_issued[0], (n + 1) & 1, abort, 28)) break;
                // the real dependency: this tile's P of pair n
                if (!mbar_wait(&sh.p_full[t], n & 1, abort, 22)) break;
                tc_fence_after();
                // O_t += P_t V: P in S_t columns 0-63, 16 keys (8 columns) per k-step
                const uint64_t vds = vd + (uint64_t)((st * C::PAIR_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    umma_ts(o_tmem, s_tmem + kk * 8, vds + (uint64_t)((kk * 2048) >> 4), idesc_o,
                            (n > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&sh.pv_done[t]);
                // S_t(n+1) right behind PV_t(n): in order on the pipe, so P_t(n) is
                // read before S_t(n+1) overwrites it
                if (more) issue_s(n + 1);
            }
        }
    }
    } else {
        // -------------------------------- softmax + epilogue (warps 0-7)
        setmaxnreg_inc<C::REG_HIGH>();
        const int t = warp >> 2;
        const int r = ((warp & 3) << 5) | lane;              // row = TMEM lane
        const int tok = token0 + t * C::TOK + r / G;
        const long p = (long)q_pos0 + tok;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_addr = lane_addr + C::S_COL + 128 * t;
        const uint32_t o_addr = lane_addr + C::O_COL + 128 * t;
        const uint64_t sc2 = f2_pack(sm_scale_log2, sm_scale_log2);
        float m_run = -INFINITY, l = 0.f;
        bool ok = nblk > 0;
        for (int n = 0; ok && n < npair; n++) {
            if (!mbar_wait(&sh.s_full[t], n & 1, abort, 30)) { ok = false; break; }
            tc_fence_after();
            // the issuer's commit covers every earlier MMA of this tile: S_t(n)
            // done frees K stage n, and PV_t(n-1) (issued before it) frees V
            // stage n-1 -- the stage releases ride on this wait, at no cost to
            // the issuing thread
            if ((warp & 3) == 0 && lane == 0) {
                mbar_arrive(&sh.k_empty[n % C::NS]);
                if (n > 0) mbar_arrive(&sh.v_empty[(n - 1) % C::NS]);
            }
            // keys c <= lim[hb] of the pair's half hb are visible: only the
            // diagonal block and the copy that pads an odd last pair are masked
            int lim[2];
#pragma unroll
            for (int hb = 0; hb < 2; hb++) {
                const int bi = 2 * n + hb;
                const int blk = bi < nblk ? sh.blocks[bi] : -1;
                lim[hb] = blk < 0 ? -1 : (blk == Dg ? (int)(p - 64L * Dg) : 63);
            }
            uint32_t sr[128];
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32)
                tmem_ld32(s_addr + c0, *reinterpret_cast<uint32_t(*)[32]>(&sr[c0]));
            tmem_wait_ld();
#pragma unroll
            for (int hb = 0; hb < 2; hb++) {
                if (lim[hb] < 63) {
#pragma unroll
                    for (int c = 0; c < 64; c++)
                        if (c > lim[hb]) sr[64 * hb + c] = 0xff800000u;   // -inf
                }
            }
            // 16 independent chains of 3-input maxima (the instruction's
            // latency, not its count, sets the time), then a short tree
            float qm[16];
#pragma unroll
            for (int k = 0; k < 16; k++) qm[k] = fmaxf(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]));
#pragma unroll
            for (int c = 32; c < 128; c += 32) {
#pragma unroll
                for (int k = 0; k < 16; k++)
                    qm[k] = max3f(qm[k], __uint_as_float(sr[c + 2 * k]), __uint_as_float(sr[c + 2 * k + 1]));
            }
#pragma unroll
            for (int k = 0; k < 5; k++) qm[k] = max3f(qm[3 * k], qm[3 * k + 1], qm[3 * k + 2]);
            const float mx = fmaxf(max3f(qm[0], qm[1], qm[2]), max3f(qm[3], qm[4], qm[15])) * sm_scale_log2;
            if (n == 0) {
                m_run = mx;
            } else if (__any_sync(0xffffffffu, mx > m_run + 8.0f)) {
                const float m_new = fmaxf(m_run, mx);
                const float alpha = fast_exp2(m_run - m_new);
                // O_t is stable once PV_t(n-1) has completed
                if (!mbar_wait(&sh.pv_done[t], (n - 1) & 1, abort, 31)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; c++) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st32(o_addr + c0, o);
                }
                tmem_wait_st();
                l *= alpha;
                m_run = m_new;
            }
            // P = 2^(s*c - m), 1 of every 4 pairs on the FMA pipe, the rest on
            // MUFU; S is re-read from TMEM in 32-column chunks, one chunk ahead
            const uint64_t nm2 = f2_pack(-m_run, -m_run);
            uint64_t lacc[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; c++) {
                    const uint64_t x2 = f2_fma(
                        f2_pack(__uint_as_float(sr[c0 + 2 * c]), __uint_as_float(sr[c0 + 2 * c + 1])), sc2, nm2);
                    float p0, p1;
                    if ((c & 3) == 3) {
                        f2_unpack(exp2_poly_x2(x2), p0, p1);
                    } else {
                        float x0, x1;
                        f2_unpack(x2, x0, x1);
                        p0 = fast_exp2(x0);
                        p1 = fast_exp2(x1);
                    }
                    lacc[c & 3] = f2_add(lacc[c & 3], f2_pack(p0, p1));
                    pk[c] = pack_bf16x2(p0, p1);
                }
                // P over S columns [c0/2, c0/2 + 16): S is held in registers
                tmem_st16(s_addr + c0 / 2, pk);
            }
            float la, lb;
            f2_unpack(f2_add(f2_add(lacc[0], lacc[1]), f2_add(lacc[2], lacc[3])), la, lb);
            l += la + lb;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_full[t]);
        }
        if (ok && !mbar_wait(&sh.pv_done[t], (npair - 1) & 1, abort, 32)) ok = false;
        tc_fence_after();
        const bool store = tok < Tq;
        const int h = g * G + r % G;
        __nv_bfloat16 *orow = O + (((long)b * Tq + tok) * Hq + h) * D;
        const float inv_l = (ok && l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(o_addr + c0, o);
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
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace qsa
