// Step 5 (prefill) -- exact softmax attention over the selected blocks only
// (page "Qwen4 architecture: QSA, GR, PLE", section 1, "attend closely to
// the selected regions"; page "Qwen4 in llama.cpp: Dissecting PR #27742",
// section "QSA Is an Address-Selection Problem, Not a New Attention
// Equation": ordinary attention over the visible cells).
//
// Work unit (one CTA, one per SM): two 128-row MMA tiles of one KV group
// and query block; row r of a tile = token (r / G), query head (r % G) --
// 256 rows sharing the same selected key blocks, so every gathered K/V
// block is loaded once for all 256 rows.  One selected 64-key block per
// step, through separate 4-deep K and V rings; per block n and tile t:
//     S_t(n) = Q_t K_n^T    tcgen05.mma kind::f16, M=128 N=64 K=16 steps,
//                           A = Q_t, B = the block's keys (both K-major in
//                           shared memory), D = S buffer n%2 of tile t in
//                           TMEM (fp32)
//     P_t(n) = 2^(S c - m)  softmax warpgroup t, one thread per row; bf16
//                           P is written over the first 32 columns of the
//                           same S buffer
//     O_t += P_t(n) V_n     tcgen05.mma, A = P from TMEM, B = the block's
//                           values (MN-major in shared memory), D = O_t
// S is double-buffered in TMEM: the issuer of tile t puts S_t(n+2) on the
// pipe right behind PV_t(n) (the pipe runs a thread's MMAs in order, so
// PV_t(n) reads P_t(n) before S_t(n+2) overwrites it), and when the
// softmax finishes block n, S_t(n+1) is normally complete already.  Both
// tiles' softmaxes therefore run all the time, side by side on the SM's
// issue slots, while the tensor pipe works through the MMAs both tiles
// keep queued.  The running max only moves (and O_t is rescaled in TMEM)
// when a block's max exceeds it by more than 2^8.
//
// Warps (384 threads, three warpgroups): 0-7 softmax/epilogue (tile =
// warp/4, TMEM lane quarter = warp%4, thread = row), 8 TMA producer of Q
// and K, 9 TMEM allocator + MMA issuer of tile 0, 10 MMA issuer of tile 1,
// 11 TMA producer of V.  The last warpgroup gives registers to the softmax
// warpgroups (setmaxnreg).  Each softmax warp signals P with a single
// arrive, and the softmax warps release the K and V stages: an MMA commit
// covers every earlier MMA of its thread, so S_t(n) done frees K_n for
// tile t and, S_t(n) being issued behind PV_t(n-2), V_{n-2} too.
// TMEM (512 columns): O_0 [0,128) O_1 [128,256); S buffer b of tile t at
// [256 + 128t + 64b, +64), P in its first 32 columns.  Every mbarrier wait
// is bounded.
#pragma once
#include "device.cuh"

namespace qsa {

template <int D, int G>
struct PrefillCfg {
    static constexpr int M = 128;                  // rows per tile
    static constexpr int TOK = M / G;              // tokens per tile
    static constexpr int TILES = 64 / (2 * TOK);   // CTAs per 64-token query block
    static constexpr int NH = D / 64;              // 128-byte column halves
    static constexpr int Q_HALF = 128 * 128;       // 128 rows x 128 B
    static constexpr int QT_BYTES = NH * Q_HALF;   // one Q tile
    static constexpr int B_HALF = 64 * 128;        // 64 rows x 128 B
    static constexpr int BLK_BYTES = NH * B_HALF;  // K (or V) of one block
    static constexpr int NS = 4;                   // K stages and V stages (blocks)
    static constexpr int SMEM_DATA = 2 * QT_BYTES + 2 * NS * BLK_BYTES;
    // the CTA owns all 512 TMEM columns: ask for enough shared memory that
    // a second CTA never lands on the same SM
    static constexpr int SMEM_REQUEST = (SMEM_DATA + 1024 > 120 * 1024) ? SMEM_DATA + 1024 : 120 * 1024;
    static constexpr int THREADS = 12 * 32;
    // registers: launched at REG_LAUNCH per thread (the launch bounds'
    // ceiling for 384 threads, checked by the build); the producer/issuer
    // warpgroup drops to REG_LOW and the two softmax warpgroups rise to
    // REG_HIGH: 256 * REG_HIGH + 128 * REG_LOW must not exceed
    // 384 * REG_LAUNCH
    static constexpr int REG_LAUNCH = 168;
    static constexpr int REG_LOW = 48;
    static constexpr int REG_HIGH = 224;
    static_assert(256 * REG_HIGH + 128 * REG_LOW <= 384 * REG_LAUNCH, "register split exceeds the launch pool");
    static constexpr int TMEM_COLS = 512;
    static constexpr int O_COL = 0, S_COL = 256;
};

struct PrefillShared {
    uint64_t q_full;
    uint64_t k_full[4], k_empty[4];
    uint64_t v_full[4], v_empty[4];
    uint64_t s_full[2][2];      // [tile][S buffer]
    uint64_t p_full[2][2];      // [tile][S buffer]
    uint64_t pv_done[2];        // [tile]
    uint64_t stag[2];           // [tile]: its softmax has its block max
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
    uint8_t *k_smem = smem + 2 * C::QT_BYTES;        // [stage][half][64 rows][128 B]
    uint8_t *v_smem = k_smem + C::NS * C::BLK_BYTES;

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
            for (int bf = 0; bf < 2; bf++) {
                mbar_init(&sh.s_full[t][bf], 1);
                mbar_init(&sh.p_full[t][bf], 4);   // one arrive per softmax warp
            }
            mbar_init(&sh.pv_done[t], 1);
            mbar_init(&sh.stag[t], 4);
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
    volatile int *abort = &sh.abort;

    if (warp >= 8) {
    // warpgroup 2 (one setmaxnreg for its four warps): producers, issuers
    setmaxnreg_dec<C::REG_LOW>();
    if (warp == 8 || warp == 11) {
        // ---------------------------- TMA producers: Q and K (8), V (11)
        const bool is_k = warp == 8;
        if (lane == 0 && nblk > 0) {
            if (is_k) {
                mbar_arrive_expect_tx(&sh.q_full, 2 * C::QT_BYTES);
                for (int t = 0; t < 2; t++)
                    for (int h = 0; h < C::NH; h++)
                        tma_load_3d(q_smem + t * C::QT_BYTES + h * C::Q_HALF, &tmQ, &sh.q_full, h * 64,
                                    g * G, b * Tq + token0 + t * C::TOK);
            }
            const CUtensorMap *map = is_k ? &tmK : &tmV;
            uint64_t *full = is_k ? sh.k_full : sh.v_full;
            uint64_t *empty = is_k ? sh.k_empty : sh.v_empty;
            uint8_t *ring = is_k ? k_smem : v_smem;
            const int kv_row0 = bg * T_kv_max;   // host checks B*Hkv*T_kv_max < 2^31
            for (int n = 0; n < nblk; n++) {
                const int st = n % C::NS;
                if (n >= C::NS && !mbar_wait(&empty[st], ((n / C::NS) - 1) & 1, abort, is_k ? 10 : 11)) break;
                mbar_arrive_expect_tx(&full[st], C::BLK_BYTES);
                const int row = kv_row0 + 64 * sh.blocks[n];
                for (int h = 0; h < C::NH; h++)
                    tma_load_2d(ring + st * C::BLK_BYTES + h * C::B_HALF, map, &full[st], h * 64, row);
            }
        }
    } else {
        // ----------------------------------------- MMA issuer of tile t
        // the whole warp runs the loop (waits and descriptors stay
        // warp-uniform); one elected lane issues the MMAs and commits
        const int t = __shfl_sync(0xffffffffu, warp - 9, 0);
        // a wait's outcome, made warp-uniform
        auto wait_all = [&](uint64_t *bar, uint32_t parity, int where) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, where));
        };
        if (nblk > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idesc_o = umma_idesc_bf16(128, D, 0, 1);
            // descriptor bases, built once: per MMA only a 64-bit add of the
            // byte offset >> 4 into the start-address field remains (shared
            // memory addresses stay below 2^18, so the field never carries)
            const uint64_t qd = umma_smem_desc(smem_u32(q_smem + t * C::QT_BYTES), 16, 1024);
            const uint64_t kd = umma_smem_desc(smem_u32(k_smem), 16, 1024);
            const uint64_t vd = umma_smem_desc(smem_u32(v_smem), C::B_HALF, 1024);
            const uint32_t s_tmem0 = tmem + C::S_COL + 128 * t;
            const uint32_t o_tmem = tmem + C::O_COL + 128 * t;
            // S_t(n) = Q_t K_n^T into S buffer n%2
            auto issue_s = [&](int n) -> bool {
                const int st = n % C::NS;
                if (!wait_all(&sh.k_full[st], (n / C::NS) & 1, 21)) return false;
                tc_fence_after();
                const uint64_t kds = kd + (uint64_t)((st * C::BLK_BYTES) >> 4);
                const uint32_t s_tmem = s_tmem0 + 64 * (n & 1);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; kk++) {
                        const uint64_t qoff = (uint64_t)((((kk >> 2) * C::Q_HALF) + (kk & 3) * 32) >> 4);
                        const uint64_t koff = (uint64_t)((((kk >> 2) * C::B_HALF) + (kk & 3) * 32) >> 4);
                        umma_ss(s_tmem, qd + qoff, kds + koff, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&sh.s_full[t][n & 1]);
                }
                __syncwarp();
                return true;
            };
            bool ok = wait_all(&sh.q_full, 0, 20);
            if (ok) ok = issue_s(0);
            if (ok && nblk > 1) ok = issue_s(1);
            for (int n = 0; ok && n < nblk; n++) {
                const int st = n % C::NS;
                if (!wait_all(&sh.v_full[st], (n / C::NS) & 1, 26)) break;
                // the real dependency: this tile's P of block n
                if (!wait_all(&sh.p_full[t][n & 1], (n >> 1) & 1, 22)) break;
                tc_fence_after();
                // O_t += P_t V: P in the S buffer's columns 0-31, 16 keys
                // (8 columns) per k-step
                const uint64_t vds = vd + (uint64_t)((st * C::BLK_BYTES) >> 4);
                const uint32_t p_tmem = s_tmem0 + 64 * (n & 1);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        umma_ts(o_tmem, p_tmem + kk * 8, vds + (uint64_t)((kk * 2048) >> 4), idesc_o,
                                (n > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sh.pv_done[t]);
                }
                __syncwarp();
                // S_t(n+2) into the same buffer, right behind PV_t(n)
                if (n + 2 < nblk && !issue_s(n + 2)) break;
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
        const uint32_t s_addr0 = lane_addr + C::S_COL + 128 * t;
        const uint32_t o_addr = lane_addr + C::O_COL + 128 * t;
        const uint64_t sc2 = f2_pack(sm_scale_log2, sm_scale_log2);
        float m_run = -INFINITY, l = 0.f;
        bool ok = nblk > 0;
        for (int n = 0; ok && n < nblk; n++) {
            // stagger: tile 1 starts block n once tile 0 has the max of n,
            // tile 0 starts block n once tile 1 has the max of n-1, so one
            // tile's loads and max run during the other's exponentials
            if (t == 1 || n > 0) {
                if (!mbar_wait(&sh.stag[t ^ 1], (n - (t ^ 1)) & 1, abort, 33)) { ok = false; break; }
            }
            if (!mbar_wait(&sh.s_full[t][n & 1], (n >> 1) & 1, abort, 30)) { ok = false; break; }
            tc_fence_after();
            // the issuer's commit covers every earlier MMA of this tile: S_t(n)
            // done frees K stage n and, PV_t(n-2) having been issued before
            // it, V stage n-2 -- the stage releases ride on this wait
            if ((warp & 3) == 0 && lane == 0) {
                mbar_arrive(&sh.k_empty[n % C::NS]);
                if (n >= 2) mbar_arrive(&sh.v_empty[(n - 2) % C::NS]);
            }
            const uint32_t s_addr = s_addr0 + 64 * (n & 1);
            // keys c <= lim of the block are visible: only the diagonal
            // block is masked
            const int blk = sh.blocks[n];
            const int lim = blk == Dg ? (int)(p - 64L * Dg) : 63;
            uint32_t sr[64];
            tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
            if (lim < 63) {
#pragma unroll
                for (int c = 0; c < 64; c++)
                    if (c > lim) sr[c] = 0xff800000u;   // -inf
            }
            // 16 independent chains of 3-input maxima (the instruction's
            // latency, not its count, sets the time), then a short tree
            float qm[16];
#pragma unroll
            for (int k = 0; k < 16; k++)
                qm[k] = max3f(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]),
                              __uint_as_float(sr[32 + 2 * k]));
#pragma unroll
            for (int k = 0; k < 16; k++) qm[k] = fmaxf(qm[k], __uint_as_float(sr[33 + 2 * k]));
#pragma unroll
            for (int k = 0; k < 5; k++) qm[k] = max3f(qm[3 * k], qm[3 * k + 1], qm[3 * k + 2]);
            const float mx = fmaxf(max3f(qm[0], qm[1], qm[2]), max3f(qm[3], qm[4], qm[15])) * sm_scale_log2;
            if (lane == 0) mbar_arrive(&sh.stag[t]);
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
            // MUFU; packed bf16 P goes over the buffer's first 32 columns
            const uint64_t nm2 = f2_pack(-m_run, -m_run);
            uint64_t lacc[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
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
            if (lane == 0) mbar_arrive(&sh.p_full[t][n & 1]);
        }
        if (ok && !mbar_wait(&sh.pv_done[t], (nblk - 1) & 1, abort, 32)) ok = false;
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
