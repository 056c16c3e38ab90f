// Step 5 (prefill) -- exact softmax attention over the selected blocks only
// (page "Qwen4 architecture: QSA, GR, PLE", section 1, "attend closely to
// the selected regions"; page "Qwen4 in llama.cpp: Dissecting PR #27742",
// section "QSA Is an Address-Selection Problem, Not a New Attention
// Equation": ordinary attention over the visible cells).
//
// Persistent kernel: one CTA per SM walks the work units u = blockIdx.x,
// blockIdx.x + gridDim.x, ...  A unit is two 128-row MMA tiles of one KV
// group and query block; row r of a tile = token (r / G), query head
// (r % G) -- 256 rows sharing the same selected key blocks, so every
// gathered K/V block is loaded once for all 256 rows.  The CTA treats the
// blocks of all its units as one stream (ring stages, S buffers and barrier
// phases count blocks across units), so the next unit's block list, Q tiles,
// first K/V blocks and first S MMAs are on their way while the current
// unit's last blocks and epilogue run.  One selected 64-key block per step,
// through separate 4-deep K and V rings; per block n and tile t:
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
// softmax finishes block n, S_t(n+1) is normally complete already.  Tile 1
// trails tile 0 by half a block (each waits for the other's block max), so
// one tile's TMEM loads and max run during the other's exponentials while
// the tensor pipe works through the MMAs both tiles keep queued.  The
// running max only moves (and O_t is rescaled in TMEM) when a block's max
// exceeds it by more than 2^8.  At a unit boundary the issuer puts both
// last PVs on the pipe before the next unit's first S (which waits for the
// next Q tiles), and the next unit's first PV -- which overwrites O_t --
// waits for P of its block, which the softmax warps signal only after
// their epilogue has read O_t.
//
// Warps (384 threads, three warpgroups): 0-7 softmax/epilogue (tile =
// warp/4, TMEM lane quarter = warp%4, thread = row), 8 block-list reader
// and TMA producer of Q and K, 9 TMEM allocator + MMA issuer of tile 0,
// 10 MMA issuer of tile 1, 11 TMA producer of V.  The last warpgroup gives
// registers to the softmax warpgroups (setmaxnreg).  Each softmax warp
// signals P with a single arrive, and the softmax warps release the K and
// V stages: an MMA commit covers every earlier MMA of its thread, so S_t(n)
// done frees K_n for tile t and, S_t(n) being issued behind PV_t(n-2),
// V_{n-2} too.  The issuers' commit after a unit's last S frees the Q tiles.
// TMEM (512 columns): O_0 [0,128) O_1 [128,256); S buffer b of tile t at
// [256 + 128t + 64b, +64), P in its first 32 columns.  Every mbarrier wait
// is bounded.
//
// Ragged batches over paged caches (serving, chunked prefill of several
// requests): sequence b's chunk starts at q_pos[b] (device data) and its
// logical block j lives in page block_table[b][j] of [num_pages][Hkv][64][d].
// The list reader checks the position and every page before any load
// (QSA_ERR_BOUNDS) and hands the producers each block's first cache row.
#pragma once
#include "device.cuh"

namespace qsa {

template <int D, int G>
struct PrefillCfg {
    static constexpr int M = 128;                  // rows per tile
    static constexpr int TOK = M / G;              // tokens per tile
    static constexpr int TILES = 64 / (2 * TOK);   // units per 64-token query block
    static constexpr int NH = D / 64;              // 128-byte column halves
    static constexpr int Q_HALF = 128 * 128;       // 128 rows x 128 B
    static constexpr int QT_BYTES = NH * Q_HALF;   // one Q tile
    static constexpr int B_HALF = 64 * 128;        // 64 rows x 128 B
    static constexpr int BLK_BYTES = NH * B_HALF;  // K (or V) of one block
    static constexpr int NS = 4;                   // K stages and V stages (blocks)
    // epilogue staging: per softmax warp, 32 rows x 128 B (one 64-column
    // half of O at a time) for a transpose into coalesced stores
    static constexpr int STAGE_BYTES = 32 * 128;
    static constexpr int SMEM_DATA = 2 * QT_BYTES + 2 * NS * BLK_BYTES + 8 * STAGE_BYTES;
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
    static constexpr int REG_LOW = 56;
    static constexpr int REG_HIGH = 224;
    static_assert(256 * REG_HIGH + 128 * REG_LOW <= 384 * REG_LAUNCH, "register split exceeds the launch pool");
    static constexpr int TMEM_COLS = 512;
    static constexpr int O_COL = 0, S_COL = 256;
    // arrivals that free a block-list slot: V producer, two issuers, eight
    // softmax warps
    static constexpr int LIST_USERS = 11;
};

struct PrefillShared {
    uint64_t q_full, q_empty;
    uint64_t k_full[4], k_empty[4];
    uint64_t v_full[4], v_empty[4];
    uint64_t s_full[2][2];      // [tile][S buffer]
    uint64_t p_full[2][2];      // [tile][S buffer]
    uint64_t pv_done[2];        // [tile]: completes once per block (its PV)
    uint64_t o_full[2];         // [tile]: completes once per unit (its last PV)
    uint64_t stag[2];           // [tile]: its softmax has its block max
    uint64_t list_full[2], list_empty[2];   // [list slot]
    uint32_t tmem_base;
    int abort;
    int nblk[2];                // [list slot] blocks of the unit (>= 1)
    int none[2];                // [list slot] the row lists no valid block
    int qp[2];                  // [list slot] the sequence's first query position
    int diag[2];                // [list slot] the last listed block is the diagonal block
    int rows[2][64];            // [list slot] first cache row of each block (TMA coordinate)
};

// Work unit u -> query block i, first token, batch x KV group bg.  False for
// the idle units past a ragged last query block.
struct PrefillUnit {
    int i, bg, token0;
};

template <int TILES, int TOK>
__device__ __forceinline__ bool prefill_unit(int u, int NX, int Tq, PrefillUnit &w)
{
    const int x = u % NX;
    w.bg = u / NX;
    w.i = x / TILES;
    w.token0 = w.i * 64 + (x % TILES) * 2 * TOK;
    return w.token0 < Tq;
}

template <int D, int G>
__global__ void __launch_bounds__(12 * 32, 1) sparse_attn_prefill_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ idx,
    __nv_bfloat16 *__restrict__ O, float *__restrict__ lse, int Tq, int Hq, int Hkv, int BH,
    int q_pos0, int T_kv_max, int topk, float sm_scale_log2, const int32_t *__restrict__ q_pos,
    const int32_t *__restrict__ block_table, int max_blocks, int num_pages, int blk_lo, int blk_hi,
    int partial)
{
    using C = PrefillCfg<D, G>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ PrefillShared sh;

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *q_smem = smem;                          // [tile][half][128 rows][128 B]
    uint8_t *k_smem = smem + 2 * C::QT_BYTES;        // [stage][half][64 rows][128 B]
    uint8_t *v_smem = k_smem + C::NS * C::BLK_BYTES;
    uint8_t *o_stage = v_smem + C::NS * C::BLK_BYTES;   // [softmax warp][32 rows][8 x 16 B]

    const int NR = (Tq + 63) / 64;
    const int NX = NR * C::TILES;
    const int U = NX * BH;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        sh.abort = 0;
        mbar_init(&sh.q_full, 1);
        mbar_init(&sh.q_empty, 2);           // one commit per issuer
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
            mbar_init(&sh.o_full[t], 1);
            mbar_init(&sh.stag[t], 4);
            mbar_init(&sh.list_full[t], 1);
            mbar_init(&sh.list_empty[t], C::LIST_USERS);
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
    volatile int *abort = &sh.abort;
    // a wait's outcome, made warp-uniform (a warp never splits on a timeout)
    auto wait_all = [&](uint64_t *bar, uint32_t parity, int where) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, where));
    };

    if (warp >= 8) {
    // warpgroup 2 (one setmaxnreg for its four warps): producers, issuers
    setmaxnreg_dec<C::REG_LOW>();
    if (warp == 8) {
        // ------------------- block lists (whole warp), Q and K (lane 0)
        int k = 0, gk = 0;   // units and K blocks so far
        bool ok = true;
        for (int u = blockIdx.x; ok && u < U; u += gridDim.x) {
            PrefillUnit w;
            if (!prefill_unit<C::TILES, C::TOK>(u, NX, Tq, w)) continue;
            const int slot = k & 1;
            const int b = w.bg / Hkv, g = w.bg % Hkv;
            int qpos = q_pos0;
            if (q_pos) {
                qpos = __ldg(q_pos + b);
                const long cap = block_table ? 64L * max_blocks : (long)T_kv_max;
                if (qpos < 0 || (qpos & 63) || (long)qpos + Tq > cap) {
                    if (lane == 0) report(QSA_ERR_BOUNDS, 11);
                    qpos = 0;
                }
            }
            const int Dg = (qpos + min(w.i * 64 + 63, Tq - 1)) / 64;
            const long kv_row0 = (long)w.bg * T_kv_max;   // contiguous: host checks B*Hkv*T_kv_max < 2^31
            if (k >= 2 && !wait_all(&sh.list_empty[slot], ((k >> 1) - 1) & 1, 12)) break;
            // the row's list, one entry per lane: it ends at the first -1;
            // an index past the diagonal or not above its predecessor is an
            // error and ends it too.  Listed blocks outside [blk_lo, blk_hi)
            // belong to another rank's cache and are skipped; an owned
            // block j is cache block j - blk_lo of this rank.
            const int32_t *sel = idx + ((long)w.bg * NR + w.i) * topk;
            int n = 0, prev = -1, lastj = -1;
            bool bad = false;
            for (int r0 = 0; r0 < topk; r0 += 32) {
                const int s = r0 + lane;
                const int j = s < topk ? sel[s] : -1;
                int jp = __shfl_up_sync(0xffffffffu, j, 1);
                if (lane == 0) jp = prev;
                bool stop_bad = j >= 0 && (j > Dg || (s > 0 && j <= jp));
                const bool owned = j >= blk_lo && j < blk_hi;
                int row = 0;
                if (j >= 0 && !stop_bad && owned) {
                    if (block_table) {
                        const int page = __ldg(block_table + (long)b * max_blocks + j);
                        if (page < 0 || page >= num_pages) stop_bad = true;
                        else row = (page * Hkv + g) * 64;   // host checks num_pages*Hkv*64 < 2^31
                    } else {
                        row = (int)(kv_row0 + 64L * (j - blk_lo));
                    }
                }
                const unsigned stops = __ballot_sync(0xffffffffu, j < 0 || stop_bad);
                const int f = stops ? __ffs(stops) - 1 : 32;
                const bool keep = lane < f && owned;
                const unsigned kept = __ballot_sync(0xffffffffu, keep);
                if (keep) sh.rows[slot][n + __popc(kept & ((1u << lane) - 1u))] = row;
                if (kept) lastj = __shfl_sync(0xffffffffu, j, 31 - __clz(kept));
                n += __popc(kept);
                if (stops) {
                    bad = __shfl_sync(0xffffffffu, stop_bad, f);
                    break;
                }
                prev = __shfl_sync(0xffffffffu, j, 31);
            }
            if (lane == 0) {
                if (bad) report(QSA_ERR_BOUNDS, 1);
                if (n == 0) {
                    // no valid block: block 0 goes through the pipeline (in
                    // bounds) and the epilogue writes zeros -- an error,
                    // unless this rank owns none of a row's blocks (partial)
                    if (!partial) report(QSA_ERR_BOUNDS, 2);
                    lastj = 0;
                    int row0 = (int)kv_row0;
                    if (block_table) {
                        const int page = __ldg(block_table + (long)b * max_blocks);
                        row0 = (page >= 0 && page < num_pages) ? (page * Hkv + g) * 64 : 0;
                    }
                    sh.rows[slot][0] = row0;
                }
                sh.nblk[slot] = max(n, 1);
                sh.none[slot] = n == 0;
                sh.qp[slot] = qpos;
                // a valid list is ascending and ends at or before the
                // diagonal, so only its last block can be the diagonal
                sh.diag[slot] = lastj == Dg;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh.list_full[slot]);
                // Q tiles of the unit, once the previous unit's S are done
                if (k >= 1 && !mbar_wait(&sh.q_empty, (k - 1) & 1, abort, 13)) ok = false;
                if (ok) {
                    mbar_arrive_expect_tx(&sh.q_full, 2 * C::QT_BYTES);
                    for (int t = 0; t < 2; t++)
                        for (int h = 0; h < C::NH; h++)
                            tma_load_3d(q_smem + t * C::QT_BYTES + h * C::Q_HALF, &tmQ, &sh.q_full, h * 64,
                                        g * G, b * Tq + w.token0 + t * C::TOK);
                }
                for (int nn = 0; ok && nn < max(n, 1); nn++) {
                    const int gb = gk + nn, st = gb % C::NS;
                    if (gb >= C::NS && !mbar_wait(&sh.k_empty[st], ((gb / C::NS) - 1) & 1, abort, 10)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.k_full[st], C::BLK_BYTES);
                    const int row = sh.rows[slot][nn];
                    for (int h = 0; h < C::NH; h++)
                        tma_load_2d(k_smem + st * C::BLK_BYTES + h * C::B_HALF, &tmK, &sh.k_full[st], h * 64, row);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            gk += max(n, 1);
            k++;
        }
    } else if (warp == 11) {
        // --------------------------------------------- V producer (lane 0)
        if (lane == 0) {
            int k = 0, gv = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < U; u += gridDim.x) {
                PrefillUnit w;
                if (!prefill_unit<C::TILES, C::TOK>(u, NX, Tq, w)) continue;
                const int slot = k & 1;
                if (!mbar_wait(&sh.list_full[slot], (k >> 1) & 1, abort, 14)) break;
                const int nb = sh.nblk[slot];
                for (int nn = 0; nn < nb; nn++, gv++) {
                    const int st = gv % C::NS;
                    if (gv >= C::NS && !mbar_wait(&sh.v_empty[st], ((gv / C::NS) - 1) & 1, abort, 11)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.v_full[st], C::BLK_BYTES);
                    const int row = sh.rows[slot][nn];
                    for (int h = 0; h < C::NH; h++)
                        tma_load_2d(v_smem + st * C::BLK_BYTES + h * C::B_HALF, &tmV, &sh.v_full[st], h * 64, row);
                }
                mbar_arrive(&sh.list_empty[slot]);
                k++;
            }
        }
    } else {
        // ----------------------------------------- MMA issuer of tile t
        // the whole warp runs the loop (waits and descriptors stay
        // warp-uniform); one elected lane issues the MMAs and commits
        const int t = __shfl_sync(0xffffffffu, warp - 9, 0);
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
        // S_t(gb) = Q_t K_gb^T into S buffer gb%2 (gb counts blocks across
        // units); after a unit's last S, a commit frees the Q tiles
        auto issue_s = [&](int gb, bool last_of_unit, bool wait_k) -> bool {
            const int st = gb % C::NS;
            if (wait_k && !wait_all(&sh.k_full[st], (gb / C::NS) & 1, 21)) return false;
            tc_fence_after();
            const uint64_t kds = kd + (uint64_t)((st * C::BLK_BYTES) >> 4);
            const uint32_t s_tmem = s_tmem0 + 64 * (gb & 1);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; kk++) {
                    const uint64_t qoff = (uint64_t)((((kk >> 2) * C::Q_HALF) + (kk & 3) * 32) >> 4);
                    const uint64_t koff = (uint64_t)((((kk >> 2) * C::B_HALF) + (kk & 3) * 32) >> 4);
                    umma_ss(s_tmem, qd + qoff, kds + koff, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sh.s_full[t][gb & 1]);
                if (last_of_unit) umma_commit(&sh.q_empty);
            }
            __syncwarp();
            return true;
        };
        auto next_unit = [&](int u) -> int {
            PrefillUnit w;
            while (u < U && !prefill_unit<C::TILES, C::TOK>(u, NX, Tq, w)) u += gridDim.x;
            return u;
        };
        // a unit's length from its list slot, then free the slot
        auto unit_len = [&](int k, int &nb) -> bool {
            if (!wait_all(&sh.list_full[k & 1], (k >> 1) & 1, 23)) return false;
            nb = sh.nblk[k & 1];
            __syncwarp();
            if (elect_one()) mbar_arrive(&sh.list_empty[k & 1]);
            return true;
        };
        int u = next_unit(blockIdx.x);
        int k = 0, g0 = 0, nb = 0;   // unit, its first block, its length
        bool ok = u < U && unit_len(0, nb) && wait_all(&sh.q_full, 0, 20);
        if (ok) ok = issue_s(0, nb == 1, true);
        if (ok && nb > 1) ok = issue_s(1, nb == 2, true);
        // An mbarrier wait by this thread holds up its MMA issue while the
        // (short) queue of issued MMAs drains, so the checks that a block's V
        // and the K two blocks ahead have landed are made one block early,
        // while the softmax is still working on P; once P arrives, the PV and
        // the next S go out back to back.
        auto prefetch_checks = [&](int g0u, int nbu, int n) -> bool {
            if (n < nbu && !wait_all(&sh.v_full[(g0u + n) % C::NS], ((g0u + n) / C::NS) & 1, 26)) return false;
            if (n + 2 < nbu && !wait_all(&sh.k_full[(g0u + n + 2) % C::NS], ((g0u + n + 2) / C::NS) & 1, 21))
                return false;
            return true;
        };
        while (ok) {
            ok = prefetch_checks(g0, nb, 0);
            for (int n = 0; ok && n < nb; n++) {
                const int gb = g0 + n, st = gb % C::NS;
                // the real dependency: this tile's P of the block
                if (!wait_all(&sh.p_full[t][gb & 1], (gb >> 1) & 1, 22)) { ok = false; break; }
                tc_fence_after();
                // O_t (+)= P_t V: P in the S buffer's columns 0-31, 16 keys
                // (8 columns) per k-step; the unit's first block overwrites
                const uint64_t vds = vd + (uint64_t)((st * C::BLK_BYTES) >> 4);
                const uint32_t p_tmem = s_tmem0 + 64 * (gb & 1);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        umma_ts(o_tmem, p_tmem + kk * 8, vds + (uint64_t)((kk * 2048) >> 4), idesc_o,
                                (n > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sh.pv_done[t]);
                    if (n == nb - 1) umma_commit(&sh.o_full[t]);
                }
                __syncwarp();
                // S_t(gb+2) into the same buffer, right behind PV_t(gb)
                if (n + 2 < nb && !issue_s(gb + 2, n + 3 == nb, false)) ok = false;
                if (ok) ok = prefetch_checks(g0, nb, n + 1);
            }
            if (!ok) break;
            // the next unit: its length, its Q tiles, its first two S
            u = next_unit(u + gridDim.x);
            if (u >= U) break;
            k++;
            g0 += nb;
            if (!unit_len(k, nb) || !wait_all(&sh.q_full, k & 1, 20)) break;
            if (!issue_s(g0, nb == 1, true)) break;
            if (nb > 1 && !issue_s(g0 + 1, nb == 2, true)) break;
        }
    }
    } else {
        // -------------------------------- softmax + epilogue (warps 0-7)
        setmaxnreg_inc<C::REG_HIGH>();
        const int t = warp >> 2;
        const int r = ((warp & 3) << 5) | lane;              // row = TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_addr0 = lane_addr + C::S_COL + 128 * t;
        const uint32_t o_addr = lane_addr + C::O_COL + 128 * t;
        const uint64_t sc2 = f2_pack(sm_scale_log2, sm_scale_log2);
        int k = 0, g0 = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < U; u += gridDim.x) {
            PrefillUnit w;
            if (!prefill_unit<C::TILES, C::TOK>(u, NX, Tq, w)) continue;
            const int slot = k & 1;
            if (!wait_all(&sh.list_full[slot], (k >> 1) & 1, 34)) { ok = false; break; }
            const int nb = sh.nblk[slot];
            const bool none = sh.none[slot] != 0;
            const bool diag = sh.diag[slot] != 0;
            const int b = w.bg / Hkv, g = w.bg % Hkv;
            const int qpos = sh.qp[slot];
            const int Dg = (qpos + min(w.i * 64 + 63, Tq - 1)) / 64;
            const int tok = w.token0 + t * C::TOK + r / G;
            const long p = (long)qpos + tok;
            float m_run = -INFINITY, l = 0.f;
            for (int n = 0; n < nb; n++) {
                const int gb = g0 + n;
                // stagger: tile 1 starts block gb once tile 0 has its max,
                // tile 0 starts it once tile 1 has the max of gb-1
                if (t == 1 || gb > 0) {
                    if (!wait_all(&sh.stag[t ^ 1], (gb - (t ^ 1)) & 1, 33)) { ok = false; break; }
                }
                if (!wait_all(&sh.s_full[t][gb & 1], (gb >> 1) & 1, 30)) { ok = false; break; }
                tc_fence_after();
                // the issuer's commit covers every earlier MMA of this tile:
                // S_t(gb) done frees K stage gb and, PV_t(gb-2) having been
                // issued before it, V stage gb-2
                if ((warp & 3) == 0 && lane == 0) {
                    mbar_arrive(&sh.k_empty[gb % C::NS]);
                    if (gb >= 2) mbar_arrive(&sh.v_empty[(gb - 2) % C::NS]);
                }
                const uint32_t s_addr = s_addr0 + 64 * (gb & 1);
                // keys c <= lim of the block are visible: only the diagonal
                // block (the list's last, when listed) is masked
                const int lim = (n == nb - 1 && diag) ? (int)(p - 64L * Dg) : 63;
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
                for (int c = 0; c < 16; c++)
                    qm[c] = max3f(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]),
                                  __uint_as_float(sr[32 + 2 * c]));
#pragma unroll
                for (int c = 0; c < 16; c++) qm[c] = fmaxf(qm[c], __uint_as_float(sr[33 + 2 * c]));
#pragma unroll
                for (int c = 0; c < 5; c++) qm[c] = max3f(qm[3 * c], qm[3 * c + 1], qm[3 * c + 2]);
                const float mx = fmaxf(max3f(qm[0], qm[1], qm[2]), max3f(qm[3], qm[4], qm[15])) * sm_scale_log2;
                if (lane == 0) mbar_arrive(&sh.stag[t]);
                if (n == 0) {
                    m_run = mx;
                } else if (__any_sync(0xffffffffu, mx > m_run + 8.0f)) {
                    const float m_new = fmaxf(m_run, mx);
                    const float alpha = fast_exp2(m_run - m_new);
                    // O_t is stable once PV_t(gb-1) has completed
                    if (!wait_all(&sh.pv_done[t], (gb - 1) & 1, 31)) { ok = false; break; }
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
                // P = 2^(s*c - m), 1 of every 16 pairs on the FMA pipe (the
                // share that measured fastest with both tiles' softmaxes on
                // the SM), the rest on MUFU; packed bf16 P goes over the
                // buffer's first 32 columns
                const uint64_t nm2 = f2_pack(-m_run, -m_run);
                uint64_t lacc[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; c++) {
                        const uint64_t x2 = f2_fma(
                            f2_pack(__uint_as_float(sr[c0 + 2 * c]), __uint_as_float(sr[c0 + 2 * c + 1])), sc2,
                            nm2);
                        float p0, p1;
                        if ((c & 15) == 15) {
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
                if (lane == 0) mbar_arrive(&sh.p_full[t][gb & 1]);
            }
            if (!ok) break;
            if (lane == 0) mbar_arrive(&sh.list_empty[slot]);
            // epilogue: O_t / l once the unit's last PV is done.  That is
            // the unit's own barrier (one phase per unit): pv_done counts
            // blocks, and here only PV(g0 + nb - 3) is known to be done, so
            // its parity could not tell PV(g0 + nb - 1) from PV(g0 + nb - 3).
            // The next unit's first PV overwrites O_t only after P of its
            // block, which this warp signals after these loads.
            if (!wait_all(&sh.o_full[t], k & 1, 32)) { ok = false; break; }
            tc_fence_after();
            const float inv_l = (!none && l > 0.f) ? 1.0f / l : 0.f;
            // O_t / l as bf16, one 64-column half at a time: each thread
            // puts its row into the warp's staging rows (16-byte chunk c of
            // row rr at chunk c ^ (rr % 8), so that both the row-wise writes
            // and the column-wise reads below are free of bank conflicts),
            // then every store instruction writes four whole 128-byte rows
            uint4 *stage = reinterpret_cast<uint4 *>(o_stage + warp * C::STAGE_BYTES);
#pragma unroll
            for (int hh = 0; hh < C::NH; hh++) {
                uint32_t o[64];
                tmem_ld32(o_addr + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                tmem_ld32(o_addr + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; e++)
                        pk[e] = pack_bf16x2(__uint_as_float(o[8 * c + 2 * e]) * inv_l,
                                            __uint_as_float(o[8 * c + 2 * e + 1]) * inv_l);
                    stage[lane * 8 + (c ^ (lane & 7))] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    const int rr = 4 * q + (lane >> 3), c = lane & 7;
                    const uint4 v = stage[rr * 8 + (c ^ (rr & 7))];
                    const int row = ((warp & 3) << 5) + rr;     // tile row
                    const int tk = w.token0 + t * C::TOK + row / G;
                    if (tk < Tq)
                        reinterpret_cast<uint4 *>(O + (((long)b * Tq + tk) * Hq + g * G + row % G) * D + hh * 64)[c] = v;
                }
                __syncwarp();
            }
            const bool store = tok < Tq;
            const int h = g * G + r % G;
            if (store && lse)
                lse[((long)b * Tq + tok) * Hq + h] =
                    (!none && l > 0.f) ? (m_run + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            g0 += nb;
            k++;
        }
        if (!ok) *abort = 1;   // a wait gave up: let the other roles' waits end at once
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace qsa
