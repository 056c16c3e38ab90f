// Step 3 for prefill rows under the max-over-tokens and softmax-sum
// aggregators.  Max: the score of candidate block j for query block i is
// the largest, over the block's tokens t, of the group's head mean of
// sm_scale <q_{h,t}, Kc_j>.  The pages
// have the selector score compressed keys against the queries (page "Qwen4
// in llama.cpp: Dissecting PR #27742", section "QSA Is an Address-Selection
// Problem, Not a New Attention Equation") and leave the combination of the
// block's tokens and heads open.
//
// Unlike the pooled-query score (one dot per block and row), this needs
// every (head, token) logit: 64 x G rows against every candidate, a dense
// contraction (0.55 TFLOP over the rows of a 131072-token prefill with 16
// query heads), so it runs on the
// tensor cores.  The summaries are the bf16 option's (exact bf16 products,
// fp32 accumulation in TMEM).  The candidates sit on the MMA's M side (128
// per tile, one TMEM lane each) and the query rows (token, head) on N, so
// each epilogue thread reduces its own candidate's row: the head sum of
// every token, then the maximum over the block's valid tokens -- no
// shuffles.
//
// Both aggregators' candidate scores come from one persistent kernel body
// (block_scores_body: candidate tiles streamed through a TMA ring, tcgen05
// MMAs into two TMEM accumulators, 16 epilogue warps reducing them); scores
// go to a table [B][Hkv][NR][nblk_max] (candidates 1 .. D-1 of each row),
// and the chunked selection turns the table into indices.
//
// The softmax-sum aggregator (s_j = sum over the block's (head, token) rows
// of each row's softmax over the blocks 0 .. D-1, at j) takes two passes,
// both persistent (one CTA per SM) with 16 epilogue warps (four per TMEM
// lane quarter, 64 columns each, the ranges meeting in shared memory):
// block_softmax_stats_kernel puts the (head, token) rows on M and the blocks
// on N -- the shape of an attention score tile -- so that every thread keeps
// its row's running (max, sum) in base 2; then block_softmax_scores_kernel
// forms, per candidate, the sum of 2^(z - max) / sum over the rows, with the
// rows' statistics in shared memory.
#pragma once

#include "device.cuh"

namespace qsa {

// The softmax-sum passes evaluate one exponential pair in kPolyEvery with
// the degree-5 polynomial on the FMA pipe (exp2_poly5_x2) and the rest on
// MUFU, whose issue queue bounds both passes.
constexpr int kPolyEvery = 4;
__host__ __device__ constexpr bool poly_pair(int q) { return q % kPolyEvery == kPolyEvery - 1; }

// First pass of the softmax-sum: per (token, head) row of the query block,
// the base-2 (max, sum of 2^(z - max)) of z = sm_scale log2(e) <q, Kc_j>
// over the blocks j in 0 .. D-1.  A work unit is (sequence and group, query
// block, 128-row M tile of 128/G tokens x G heads); the blocks stream
// through it in N tiles of 256.  Persistent: one CTA per SM walks the units
// u = blockIdx.x + n * gridDim.x (the query blocks with the most blocks
// first) as one stream -- the K ring, the two TMEM accumulators and their
// barriers count tiles across units, and the M tile's queries sit in one of
// two slots, so the next unit's queries and first tiles load while the
// current unit's last tiles are reduced.  Warp roles as in
// block_max_scores_kernel (producer, issuer, 16 epilogue warps, four per
// TMEM lane quarter, each on a quarter of every tile's columns).  Output:
// stats[(bg*NR + i)][64*G][2], row (token, head) = t_local*G + h.
template <int G>
struct SoftmaxStatsCfg {
    static constexpr int D = 128;
    static constexpr int M = 128;                       // (token, head) rows per unit
    static constexpr int N = 256;                       // blocks per tile
    static constexpr int TOKM = M / G;                  // tokens per unit
    static constexpr int NMT = 64 / TOKM;               // M tiles per query block
    static constexpr int QHALF_BYTES = M * 128;         // 16 KB
    static constexpr int Q_BYTES = 2 * QHALF_BYTES;     // one slot
    static constexpr int KHALF_BYTES = N * 128;         // 32 KB
    static constexpr int KSTAGE_BYTES = 2 * KHALF_BYTES;
    static constexpr int NS = 2;
    static constexpr int SMEM_BYTES = 2 * Q_BYTES + NS * KSTAGE_BYTES + 1024;
    static constexpr int SPLIT = 4;                     // epilogue warps per TMEM lane quarter
    static constexpr int EPI = 4 * SPLIT;
    static constexpr int THREADS = 64 + 32 * EPI;       // producer, issuer, epilogue warps
    static constexpr int TMEM_COLS = 2 * N;
};

template <int G>
__global__ void __launch_bounds__(SoftmaxStatsCfg<G>::THREADS, 1) block_softmax_stats_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
    float *__restrict__ stats, int Tq, int q_pos0, int nblk_max, int Hkv, float sm_scale, int NR, int nunits)
{
    using C = SoftmaxStatsCfg<G>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t q_full[2], q_empty[2], k_full[C::NS], k_empty[C::NS], t_full[2], t_empty[2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag, issued_q, issued_k, issued_mma;
    __shared__ float xm[2][C::SPLIT - 1][128], xs[2][C::SPLIT - 1][128];   // the column ranges meet here (slot = unit parity)

    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *q_smem = base;                             // two slots
    uint8_t *k_smem = base + 2 * C::Q_BYTES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // unit u -> (bg, i, mt) and the row's diagonal block Dg (blocks 0 .. Dg-1
    // normalise); units with Dg < 2 have no candidate and are skipped by
    // every role alike
    auto unit = [&](int u, int &bg, int &i, int &mt) -> int {
        const int per = NR * C::NMT;
        bg = u / per;
        const int rem = u - bg * per;
        i = NR - 1 - rem / C::NMT;
        mt = rem % C::NMT;
        return (q_pos0 + min((i + 1) * 64, Tq) - 1) / 64;
    };

    if (threadIdx.x == 0) {
        abort_flag = 0;
        issued_q = 0;
        issued_k = 0;
        issued_mma = 0;
#pragma unroll
        for (int s = 0; s < 2; s++) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], C::EPI);
        }
#pragma unroll
        for (int s = 0; s < C::NS; s++) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    volatile int *abort = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int kt = 0, un = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                int bg, i, mt;
                const int Dg = unit(u, bg, i, mt);
                if (Dg < 2) continue;
                const int b = bg / Hkv, g = bg % Hkv, qs = un & 1;
                if (un >= 2 && !mbar_wait(&q_empty[qs], ((un >> 1) - 1) & 1, abort, 88)) break;
                mbar_arrive_expect_tx(&q_full[qs], C::Q_BYTES);
#pragma unroll
                for (int h = 0; h < 2; h++)
                    tma_load_3d(q_smem + qs * C::Q_BYTES + h * C::QHALF_BYTES, &tmQ, &q_full[qs], h * 64, g * G,
                                b * Tq + i * 64 + mt * C::TOKM);
                un++;
                const int ntiles = (Dg + C::N - 1) / C::N;
                for (int k = 0; k < ntiles; k++, kt++) {
                    const int st = kt % C::NS;
                    if (kt >= C::NS && !mbar_wait(&k_empty[st], ((kt / C::NS) - 1) & 1, abort, 80)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(&k_full[st], C::KSTAGE_BYTES);
                    const int row = bg * nblk_max + C::N * k;   // host checks B*Hkv*nblk_max < 2^31
#pragma unroll
                    for (int h = 0; h < 2; h++)
                        tma_load_2d(k_smem + st * C::KSTAGE_BYTES + h * C::KHALF_BYTES, &tmKc, &k_full[st], h * 64, row);
                }
            }
            issued_q = un;
            issued_k = kt;
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer (whole warp)
        constexpr uint32_t idesc = umma_idesc_bf16(C::M, C::N, 0, 0);
        const uint64_t kd = umma_smem_desc(smem_u32(k_smem), 16, 1024);
        auto wait_all = [&](uint64_t *bar, uint32_t parity, int where) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, where));
        };
        int kt = 0, un = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            int bg, i, mt;
            const int Dg = unit(u, bg, i, mt);
            if (Dg < 2) continue;
            const int qs = un & 1;
            if (!wait_all(&q_full[qs], (un >> 1) & 1, 81)) break;
            const uint64_t qd = umma_smem_desc(smem_u32(q_smem + qs * C::Q_BYTES), 16, 1024);
            const int ntiles = (Dg + C::N - 1) / C::N;
            for (int k = 0; k < ntiles; k++) {
                const int st = kt % C::NS, buf = kt & 1;
                if (!wait_all(&k_full[st], (kt / C::NS) & 1, 82) ||
                    (kt >= 2 && !wait_all(&t_empty[buf], ((kt >> 1) - 1) & 1, 83))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < C::D / 16; kk++) {
                        const uint64_t aoff = (uint64_t)(((kk >> 2) * C::QHALF_BYTES + (kk & 3) * 32) >> 4);
                        const uint64_t boff = (uint64_t)((st * C::KSTAGE_BYTES + (kk >> 2) * C::KHALF_BYTES + (kk & 3) * 32) >> 4);
                        umma_ss(tmem + buf * C::N, qd + aoff, kd + boff, idesc, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&t_full[buf]);
                    umma_commit(&k_empty[st]);
                }
                __syncwarp();
                kt++;
            }
            if (!ok) break;
            // the slot's queries are free once the unit's MMAs are done
            if (elect_one()) umma_commit(&q_empty[qs]);
            __syncwarp();
            un++;
        }
        if (lane == 0) issued_mma = kt;
    } else {
        // ------------------------------------------- epilogue (warps 2-9)
        const int quarter = warp & 3;
        const int part = (warp - 2) >> 2;              // the range of each tile's blocks it takes
        const int r = 32 * quarter + lane;             // (token, head) row of the M tile
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float sc2 = sm_scale * 1.4426950408889634f;
        const uint64_t s2 = f2_pack(sc2, sc2);
        int kt = 0, un = 0;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
            int bg, i, mt;
            const int Dg = unit(u, bg, i, mt);
            if (Dg < 2) continue;
            const int ntiles = (Dg + C::N - 1) / C::N;
            float m_run = -INFINITY, s_run = 0.f;
            // a failed wait (an abort, after which every wait returns at
            // once) skips the work but not the exchange below: all
            // epilogue warps reach the same named barriers
            bool ok = true;
            for (int k = 0; k < ntiles; k++, kt++) {
                const int buf = kt & 1;
                ok = ok && __all_sync(0xffffffffu, mbar_wait(&t_full[buf], (kt >> 1) & 1, abort, 84));
                if (!ok) continue;
                tc_fence_after();
                // the warp's 64 columns: both 32-column loads in flight, one
                // wait, one online-softmax step
                static_assert(C::N / C::SPLIT == 64, "two TMEM loads per epilogue warp");
                const int c = part * 64;
                const int j0 = C::N * k + c;            // block of column 0 of this range (uniform)
                if (j0 < Dg) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tmem + lane_base + buf * C::N + c, v0);
                    tmem_ld32(tmem + lane_base + buf * C::N + c + 32, v1);
                    tmem_wait_ld();
                    float x0[32], x1[32];
#pragma unroll
                    for (int e = 0; e < 32; e++) {
                        x0[e] = __uint_as_float(v0[e]);
                        x1[e] = __uint_as_float(v1[e]);
                    }
                    if (j0 + 64 > Dg) {
#pragma unroll
                        for (int e = 0; e < 32; e++) {
                            if (j0 + e >= Dg) x0[e] = -INFINITY;   // 2^(-inf) = 0 below
                            if (j0 + 32 + e >= Dg) x1[e] = -INFINITY;
                        }
                    }
                    // sc2 > 0, so the largest scaled logit is the largest raw
                    // one scaled (rounding preserves the order); column j0 is
                    // valid, so mn is finite
                    const float mn = fmaxf(m_run, fmaxf(max32(x0), max32(x1)) * sc2);
                    const uint64_t nm2 = f2_pack(-mn, -mn);
                    uint64_t acc2 = f2_pack(0.f, 0.f);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        // pairs q = e (x0) and e + 1 (x1); one in kPolyEvery on the FMA pipe
                        acc2 = f2_add(acc2, exp2_pair(poly_pair(e), f2_fma(f2_pack(x0[e], x0[e + 1]), s2, nm2)));
                        acc2 = f2_add(acc2, exp2_pair(poly_pair(e + 1), f2_fma(f2_pack(x1[e], x1[e + 1]), s2, nm2)));
                    }
                    float c0, c1;
                    f2_unpack(acc2, c0, c1);
                    s_run = s_run * fast_exp2(m_run - mn) + (c0 + c1);
                    m_run = mn;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&t_empty[buf]);
            }
            // the column ranges of each row meet: rows of one TMEM lane
            // quarter involve only that quarter's four warps, so they meet at
            // the quarter's own barrier (ids 2-5); the slot alternates with
            // the unit, so the next unit's writes cannot overtake this read
            const int xslot = un & 1;
            if (part > 0) xm[xslot][part - 1][r] = m_run, xs[xslot][part - 1][r] = s_run;
            named_barrier_sync(2 + quarter, 32 * C::SPLIT);
            if (part == 0 && ok) {
                float mn = m_run;
#pragma unroll
                for (int q = 0; q < C::SPLIT - 1; q++) mn = fmaxf(mn, xm[xslot][q][r]);
                float sum = 0.f;
                if (mn != -INFINITY) {
                    sum = s_run * fast_exp2(m_run - mn);
#pragma unroll
                    for (int q = 0; q < C::SPLIT - 1; q++) sum += xs[xslot][q][r] * fast_exp2(xm[xslot][q][r] - mn);
                }
                float *out = stats + (((long)bg * NR + i) * (64 * G) + mt * C::M + r) * 2;
                out[0] = mn;
                out[1] = sum;
            }
            un++;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (abort_flag && threadIdx.x == 0) {
        // a wait gave up: let the copies and MMAs still in flight finish
        // before the shared memory and TMEM go away (bounded, no abort
        // short-cut)
        for (int n = max(0, issued_q - 2); n < issued_q; n++)
            mbar_wait(&q_full[n & 1], (n >> 1) & 1, nullptr, 85, 100000000ull);
        for (int k = max(0, issued_k - C::NS); k < issued_k; k++)
            mbar_wait(&k_full[k % C::NS], (k / C::NS) & 1, nullptr, 86, 100000000ull);
        if (issued_mma > 0) {
            const int w = issued_mma - 1;
            mbar_wait(&t_full[w & 1], (w >> 1) & 1, nullptr, 87, 100000000ull);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Candidate scores from the per-(head, token) logits z_rj = <q_r, Kc_j> of
// the query block's rows r = (token, head):
//   max mode      s_j = sm_scale * max over the block's valid tokens of the
//                 mean over the group's heads of z_rj;
//   SOFTMAX mode  s_j = sum over the rows of 2^(z_rj sm_scale log2(e) -
//                 (max_r + log2 sum_r)), the rows' statistics from
//                 block_softmax_stats_kernel (the softmax-sum's second pass).
// Candidates on the MMA's M side (128 per tile, one TMEM lane each) and the
// query rows on N (256 per MMA: 256/G tokens x G heads), so each epilogue
// thread reduces its own candidate's columns.
// Persistent: one CTA per SM walks the (sequence and group, query block)
// units, the query blocks with the most candidates first; a unit runs as
// NT sub-units, one per 256-row N tile, each streaming the unit's candidate
// tiles (the tiles are read from L2 once per sub-unit).  The sub-units'
// query tiles sit in two slots, so the next sub-unit's queries load while
// the current one is reduced; the K ring, the two TMEM accumulators and
// their barriers count tiles across sub-units.  Each candidate's sub-unit
// partials meet in the score table: the thread that owns the candidate
// stores the first and folds in the others in order (same thread, so no
// atomics and a fixed order; the max mode's maximum is order-free anyway).
// 16 epilogue warps (four per TMEM lane quarter, 64 columns each); in the
// SOFTMAX mode the next unit's row statistics are fetched while the
// current unit is reduced.
template <int G>
struct TokenScoresCfg {
    static constexpr int D = 128;
    static constexpr int M = 128;                       // candidates per tile (TMEM lanes)
    static constexpr int N = 256;                       // query rows (token, head) per MMA
    static constexpr int TOKN = N / G;                  // tokens per sub-unit
    static constexpr int NT = 64 / TOKN;                // sub-units per 64-token query block
    static constexpr int QHALF_BYTES = N * 128;         // one 64-column half (32 KB)
    static constexpr int QTILE_BYTES = 2 * QHALF_BYTES; // one slot
    static constexpr int KHALF_BYTES = M * 128;         // 16 KB
    static constexpr int KSTAGE_BYTES = 2 * KHALF_BYTES;
    static constexpr int NS = 2;
    static constexpr int SMEM_BYTES = 2 * QTILE_BYTES + NS * KSTAGE_BYTES + 1024;
    static constexpr int SPLIT = 4;                     // epilogue warps per TMEM lane quarter
    static constexpr int EPI = 4 * SPLIT;
    static constexpr int THREADS = 64 + 32 * EPI;
    static constexpr int TMEM_COLS = 2 * N;
    static constexpr int ROWS = 64 * G;                 // (token, head) rows of a query block
    static_assert(N / SPLIT == 64, "two TMEM loads per epilogue warp");
    static_assert(ROWS <= 32 * EPI, "one statistics row per epilogue thread");
};

template <int G, bool SOFTMAX>
__device__ __forceinline__ void block_scores_body(const CUtensorMap &tmQ, const CUtensorMap &tmKc,
                                                  float *__restrict__ scores, const float *__restrict__ stats,
                                                  int Tq, int q_pos0, int nblk_max, int Hkv, float sm_scale,
                                                  int NR, int nunits)
{
    using C = TokenScoresCfg<G>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t q_full[2], q_empty[2], k_full[C::NS], k_empty[C::NS], t_full[2], t_empty[2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag, issued_q, issued_k, issued_mma;
    __shared__ __align__(16) float nrstat[SOFTMAX ? 2 : 1][SOFTMAX ? C::ROWS : 4];   // SOFTMAX: -(max + log2 sum) per row (slot = unit parity)
    __shared__ float xch[2][C::SPLIT - 1][128];         // the column ranges' partials (slot = tile parity)

    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *q_smem = base;                             // two slots
    uint8_t *k_smem = base + 2 * C::QTILE_BYTES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // unit u -> (bg, i); returns the number of candidate tiles (0: no
    // candidate, the unit is skipped by every role alike)
    auto unit = [&](int u, int &bg, int &i, int &Dg) -> int {
        bg = u / NR;
        i = NR - 1 - (u - bg * NR);
        Dg = (q_pos0 + min((i + 1) * 64, Tq) - 1) / 64;   // the row's diagonal block
        return (max(Dg - 1, 0) + C::M - 1) / C::M;          // candidates 1 .. Dg-1
    };

    if (threadIdx.x == 0) {
        abort_flag = 0;
        issued_q = 0;
        issued_k = 0;
        issued_mma = 0;
#pragma unroll
        for (int s = 0; s < 2; s++) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], C::EPI);
        }
#pragma unroll
        for (int s = 0; s < C::NS; s++) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    volatile int *abort = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int kt = 0, sq = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                int bg, i, Dg;
                const int ntiles = unit(u, bg, i, Dg);
                if (ntiles == 0) continue;
                const int b = bg / Hkv, g = bg % Hkv;
                for (int nt = 0; ok && nt < C::NT; nt++) {
                    const int qs = sq & 1;
                    if (sq >= 2 && !mbar_wait(&q_empty[qs], ((sq >> 1) - 1) & 1, abort, 90)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&q_full[qs], C::QTILE_BYTES);
#pragma unroll
                    for (int h = 0; h < 2; h++)
                        tma_load_3d(q_smem + qs * C::QTILE_BYTES + h * C::QHALF_BYTES, &tmQ, &q_full[qs], h * 64,
                                    g * G, b * Tq + i * 64 + nt * C::TOKN);
                    sq++;
                    for (int k = 0; k < ntiles; k++, kt++) {
                        const int st = kt % C::NS;
                        if (kt >= C::NS && !mbar_wait(&k_empty[st], ((kt / C::NS) - 1) & 1, abort, 91)) {
                            ok = false;
                            break;
                        }
                        fence_proxy_async_smem();
                        mbar_arrive_expect_tx(&k_full[st], C::KSTAGE_BYTES);
                        const int row = bg * nblk_max + 1 + C::M * k;   // host checks B*Hkv*nblk_max < 2^31
#pragma unroll
                        for (int h = 0; h < 2; h++)
                            tma_load_2d(k_smem + st * C::KSTAGE_BYTES + h * C::KHALF_BYTES, &tmKc, &k_full[st], h * 64,
                                        row);
                    }
                }
            }
            issued_q = sq;
            issued_k = kt;
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer (whole warp)
        constexpr uint32_t idesc = umma_idesc_bf16(C::M, C::N, 0, 0);
        const uint64_t kd = umma_smem_desc(smem_u32(k_smem), 16, 1024);
        auto wait_all = [&](uint64_t *bar, uint32_t parity, int where) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, where));
        };
        int kt = 0, sq = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
            int bg, i, Dg;
            const int ntiles = unit(u, bg, i, Dg);
            if (ntiles == 0) continue;
            for (int nt = 0; ok && nt < C::NT; nt++) {
                const int qs = sq & 1;
                if (!wait_all(&q_full[qs], (sq >> 1) & 1, 92)) {
                    ok = false;
                    break;
                }
                const uint64_t qd = umma_smem_desc(smem_u32(q_smem + qs * C::QTILE_BYTES), 16, 1024);
                for (int k = 0; k < ntiles; k++) {
                    const int st = kt % C::NS, buf = kt & 1;
                    if (!wait_all(&k_full[st], (kt / C::NS) & 1, 93) ||
                        (kt >= 2 && !wait_all(&t_empty[buf], ((kt >> 1) - 1) & 1, 94))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < C::D / 16; kk++) {
                            const uint64_t aoff = (uint64_t)((st * C::KSTAGE_BYTES + (kk >> 2) * C::KHALF_BYTES + (kk & 3) * 32) >> 4);
                            const uint64_t boff = (uint64_t)(((kk >> 2) * C::QHALF_BYTES + (kk & 3) * 32) >> 4);
                            umma_ss(tmem + buf * C::N, kd + aoff, qd + boff, idesc, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&t_full[buf]);
                        umma_commit(&k_empty[st]);
                    }
                    __syncwarp();
                    kt++;
                }
                if (!ok) break;
                // the slot's queries are free once the sub-unit's MMAs are done
                if (elect_one()) umma_commit(&q_empty[qs]);
                __syncwarp();
                sq++;
            }
        }
        if (lane == 0) issued_mma = kt;
    } else {
        // ------------------------------------------- epilogue (warps 2-17)
        const int quarter = warp & 3;                  // the TMEM lanes this warp may access
        const int part = (warp - 2) >> 2;              // its 64 of the tile's 256 columns
        const int m = 32 * quarter + lane;             // candidate within the tile
        const int e = threadIdx.x - 64;                // epilogue thread: statistics row e
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        const float sc2 = sm_scale * 1.4426950408889634f;
        const uint64_t s2 = f2_pack(sc2, sc2);
        // 2^(z sc2 - max - log2 sum): the row's negated exponent offset
        auto offset = [](float mx, float sum) { return sum > 0.f ? -(mx + __log2f(sum)) : -INFINITY; };
        auto next_unit = [&](int u) {
            int bg, i, Dg;
            for (u += gridDim.x; u < nunits; u += gridDim.x)
                if (unit(u, bg, i, Dg) > 0) break;
            return u;
        };
        int u = next_unit(blockIdx.x - (int)gridDim.x);   // the first unit with candidates
        if (SOFTMAX && u < nunits && e < C::ROWS) {
            int bg, i, Dg;
            unit(u, bg, i, Dg);
            const float *st = stats + (((long)bg * NR + i) * C::ROWS + e) * 2;
            nrstat[0][e] = offset(st[0], st[1]);
        }
        named_barrier_sync(1, 32 * C::EPI);
        int kt = 0, un = 0;
        bool ok = true;
        for (; u < nunits; un++) {
            int bg, i, Dg;
            const int ntiles = unit(u, bg, i, Dg);
            const int slot = un & 1;
            // the next unit's statistics, in flight while this unit is reduced
            const int u2 = next_unit(u);
            float pm = 0.f, ps = 0.f;
            if (SOFTMAX && u2 < nunits && e < C::ROWS) {
                int bg2, i2, Dg2;
                unit(u2, bg2, i2, Dg2);
                const float *st = stats + (((long)bg2 * NR + i2) * C::ROWS + e) * 2;
                pm = st[0];
                ps = st[1];
            }
            float *srow = scores + ((long)bg * NR + i) * nblk_max;
            for (int nt = 0; nt < C::NT; nt++) {
                for (int k = 0; k < ntiles; k++, kt++) {
                    const int buf = kt & 1;
                    // a failed wait (an abort, after which every wait returns
                    // at once) skips the work but not the exchange below: all
                    // epilogue warps reach the same named barriers
                    ok = ok && __all_sync(0xffffffffu, mbar_wait(&t_full[buf], (kt >> 1) & 1, abort, 95));
                    uint64_t best2 = f2_pack(0.f, 0.f);   // SOFTMAX: two partial sums (even, odd columns)
                    float bmax = -INFINITY;                 // max mode: the best token so far
                    auto chunk = [&](const uint32_t (&r)[32], int c) {
#pragma unroll
                        for (int tt = 0; tt < 32 / G; tt++) {
                            const int tl = nt * C::TOKN + c / G + tt;   // token of these G columns, in the block
                            if constexpr (!SOFTMAX) {
                                float sum = 0.f;
#pragma unroll
                                for (int h = 0; h < G; h++) sum += __uint_as_float(r[tt * G + h]);
                                if (i * 64 + tl < Tq) bmax = fmaxf(bmax, sum);
                            } else if (i * 64 + tl < Tq) {
#pragma unroll
                                for (int h = 0; h < G; h += 4) {
                                    const float4 ns = *reinterpret_cast<const float4 *>(&nrstat[slot][tl * G + h]);
                                    const uint64_t a = f2_fma(f2_pack(__uint_as_float(r[tt * G + h]),
                                                                      __uint_as_float(r[tt * G + h + 1])),
                                                              s2, f2_pack(ns.x, ns.y));
                                    const uint64_t bb = f2_fma(f2_pack(__uint_as_float(r[tt * G + h + 2]),
                                                                       __uint_as_float(r[tt * G + h + 3])),
                                                               s2, f2_pack(ns.z, ns.w));
                                    // pairs q and q + 1 of the chunk; one in kPolyEvery on the FMA pipe
                                    best2 = f2_add(best2, exp2_pair(poly_pair((tt * G + h) / 2), a));
                                    best2 = f2_add(best2, exp2_pair(poly_pair((tt * G + h) / 2 + 1), bb));
                                }
                            }
                        }
                    };
                    if (ok) {
                        tc_fence_after();
                        const int c = part * 64;
                        uint32_t r0[32], r1[32];
                        tmem_ld32(tmem + lane_base + buf * C::N + c, r0);
                        tmem_ld32(tmem + lane_base + buf * C::N + c + 32, r1);
                        tmem_wait_ld();
                        chunk(r0, c);
                        chunk(r1, c + 32);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&t_empty[buf]);
                    }
                    // the column ranges of each candidate meet, at the barrier
                    // of its TMEM lane quarter (slot = tile parity: the writes
                    // for tile kt+2 follow the quarter's barrier of tile
                    // kt+1, which the reader passes after this read)
                    float best = bmax;
                    if constexpr (SOFTMAX) {
                        float e0, e1;
                        f2_unpack(best2, e0, e1);
                        best = e0 + e1;
                    }
                    const int xs = kt & 1;
                    if (part > 0) xch[xs][part - 1][m] = best;
                    named_barrier_sync(2 + quarter, 32 * C::SPLIT);   // the quarter's four warps
                    const int j = 1 + C::M * k + m;
                    if (part == 0 && ok && j < Dg) {
                        if constexpr (SOFTMAX) {
#pragma unroll
                            for (int q = 0; q < C::SPLIT - 1; q++) best += xch[xs][q][m];
                            // sub-unit 0 stores, the later ones add (same thread)
                            srow[j] = nt == 0 ? best : srow[j] + best;
                        } else {
#pragma unroll
                            for (int q = 0; q < C::SPLIT - 1; q++) best = fmaxf(best, xch[xs][q][m]);
                            // the head mean and the scale are monotone, so each
                            // sub-unit's scaled maximum folds in exactly
                            best = best * (1.0f / (float)G) * sm_scale;
                            srow[j] = nt == 0 ? best : fmaxf(srow[j], best);
                        }
                    }
                }
            }
            // the next unit's statistics into the other slot (its last
            // readers finished before this unit's first exchange barrier)
            if (SOFTMAX && u2 < nunits && e < C::ROWS) nrstat[slot ^ 1][e] = offset(pm, ps);
            named_barrier_sync(1, 32 * C::EPI);
            u = u2;
        }
        if (!ok) *abort = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (abort_flag && threadIdx.x == 0) {
        // a wait gave up: let the copies and MMAs still in flight finish
        // before the shared memory and TMEM go away (bounded, no abort
        // short-cut)
        for (int n = max(0, issued_q - 2); n < issued_q; n++)
            mbar_wait(&q_full[n & 1], (n >> 1) & 1, nullptr, 96, 100000000ull);
        for (int k = max(0, issued_k - C::NS); k < issued_k; k++)
            mbar_wait(&k_full[k % C::NS], (k / C::NS) & 1, nullptr, 97, 100000000ull);
        if (issued_mma > 0) {
            const int w = issued_mma - 1;
            mbar_wait(&t_full[w & 1], (w >> 1) & 1, nullptr, 98, 100000000ull);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int G>
__global__ void __launch_bounds__(TokenScoresCfg<G>::THREADS, 1) block_max_scores_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc, float *__restrict__ scores,
    int Tq, int q_pos0, int nblk_max, int Hkv, float sm_scale, int NR, int nunits)
{
    block_scores_body<G, false>(tmQ, tmKc, scores, nullptr, Tq, q_pos0, nblk_max, Hkv, sm_scale, NR, nunits);
}

template <int G>
__global__ void __launch_bounds__(TokenScoresCfg<G>::THREADS, 1) block_softmax_scores_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc, float *__restrict__ scores,
    const float *__restrict__ stats, int Tq, int q_pos0, int nblk_max, int Hkv, float sm_scale, int NR, int nunits)
{
    block_scores_body<G, true>(tmQ, tmKc, scores, stats, Tq, q_pos0, nblk_max, Hkv, sm_scale, NR, nunits);
}

}  // namespace qsa
