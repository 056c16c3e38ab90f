// Steps 2-4 -- pooled query, block scoring and top-k block selection
// ("indexer scoring" -> "top-k selection", page "Qwen4 in llama.cpp:
// Dissecting PR #27742", section "QSA Is an Address-Selection Problem, Not
// a New Attention Equation"; the selection is discontinuous at the cutoff,
// so the order is made total: score descending, then block index ascending).
//
// Kernels:
//   pool_queries_kernel  one CTA per (row, b): fp32 mean of Q over the row's
//                        tokens and each group's heads -> Qbar (workspace).
//   score_select_kernel  one CTA per (candidate chunk, row, b*Hkv): fp32
//                        scores of the chunk's block summaries into shared
//                        memory as 64-bit keys, exact radix select of the
//                        chunk's top-m, compaction in block order.  A row
//                        with one chunk writes its final indices directly;
//                        otherwise it writes its chunk's keys to the
//                        workspace.
//   merge_select_kernel  one CTA per row with several chunks: the same
//                        select over the union of the chunks' top-m lists.
//   select_token_kernel  per-token rows (qblk = 1, e.g. decode) in one
//                        launch: the chunks of a row form a thread-block
//                        cluster; every CTA pools its token's query over the
//                        group's heads, scores its chunk and pushes the
//                        chunk's top-m into the leader's shared memory; the
//                        leader selects the row.  No workspace.
// Key of candidate j with score s: (order-preserving bits of s) << 32 |
// (0xFFFFFFFF - j); keys are unique, larger = better, and the lower block
// wins a score tie.  -0.0 is folded into +0.0.
#pragma once
#include <cooperative_groups.h>

#include "device.cuh"

namespace qsa {

constexpr int kSelThreads = 256;
constexpr int kMaxChosen = 62;   // topk <= 64 minus the two forced blocks

// ------------------------------------------------------------------ pool
// grid (NR, B); blockDim = TS * NC where NC = Hq*D/8 rounded up to a warp
// (the 16-byte column chunks of a token's heads) and TS = token splits
// (TS * NC <= 1024).  Thread (s, c) sums chunk c over the tokens t0 + s,
// t0 + s + TS, ...; the TS partial sums then add in order s = 0, 1, ... and
// the group's heads fold in order -- a fixed order, so the pooled queries
// are bit-reproducible.  Splitting the tokens keeps four times the loads in
// flight for a row of few CTAs (a short chunk is latency-bound).
template <int D>
__global__ void __launch_bounds__(1024) pool_queries_kernel(const __nv_bfloat16 *__restrict__ Q,
                                                            float *__restrict__ Qbar, int Tq, int Hq, int Hkv,
                                                            int qblk, int TS)
{
    extern __shared__ float colsum[];   // [TS][Hq * D]
    const int i = blockIdx.x, b = blockIdx.y, NR = gridDim.x;
    const int nchunks = Hq * D / 8;
    const int NC = blockDim.x / TS;
    const int t = threadIdx.x % NC, sp = threadIdx.x / NC;
    const int t0 = i * qblk;
    const int t1 = min(t0 + qblk, Tq);
    if (t < nchunks) {
        const uint4 *src = reinterpret_cast<const uint4 *>(Q + ((long)b * Tq + t0) * Hq * D) + t;
        const long stride = (long)Hq * D / 8;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; e++) acc[e] = 0.f;
        int tok = t0 + sp;
        for (; tok + 3 * TS < t1; tok += 4 * TS) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; u++) v[u] = __ldg(src + (long)(tok - t0 + u * TS) * stride);
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v[u]);
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    float2 f = __bfloat1622float2(p[e]);
                    acc[2 * e] += f.x;
                    acc[2 * e + 1] += f.y;
                }
            }
        }
        for (; tok < t1; tok += TS) {
            uint4 v = __ldg(src + (long)(tok - t0) * stride);
            const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int e = 0; e < 4; e++) {
                float2 f = __bfloat1622float2(p[e]);
                acc[2 * e] += f.x;
                acc[2 * e + 1] += f.y;
            }
        }
#pragma unroll
        for (int e = 0; e < 8; e++) colsum[(long)sp * Hq * D + t * 8 + e] = acc[e];
    }
    __syncthreads();
    const int G = Hq / Hkv;
    const float inv = 1.0f / (float)((t1 - t0) * G);
    for (int o = threadIdx.x; o < Hkv * D; o += blockDim.x) {
        const int g = o / D, c = o % D;
        float sum = 0.f;
        for (int h = g * G; h < (g + 1) * G; h++) {
            float col = 0.f;
            for (int q = 0; q < TS; q++) col += colsum[(long)q * Hq * D + h * D + c];
            sum += col;
        }
        Qbar[(((long)b * Hkv + g) * NR + i) * D + c] = sum * inv;
    }
}

// ------------------------------------------------------- select helpers
__device__ __forceinline__ uint64_t make_key(float s, int j)
{
    if (s == 0.f) s = 0.f;   // -0.0 -> +0.0
    const uint32_t b = __float_as_uint(s);
    const uint32_t k = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((uint64_t)k << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
}

__device__ __forceinline__ int key_block(uint64_t key) { return (int)(0xFFFFFFFFu - (uint32_t)key); }

template <int NT>
struct SelectSharedT {
    int hist[2][256];           // digit counts, double-buffered across radix passes
    int warp_tot[NT / 32];
    int digit[2], above[2], bucket[2];
};
using SelectShared = SelectSharedT<kSelThreads>;

// Adds 1 to hist[digit] for every lane with active set (called by the
// whole warp).  When every active lane has the same digit -- the first
// passes, where a row's keys share their top digits -- one lane adds the
// count; otherwise each active lane adds its own 1 (later digits are spread
// out, so those atomics rarely collide).
__device__ __forceinline__ void hist_add(int *hist, bool active, int digit)
{
    const unsigned act = __ballot_sync(0xffffffffu, active);
    if (!act) return;
    const int lead = __ffs(act) - 1;
    const int d0 = __shfl_sync(0xffffffffu, digit, lead);
    if (__all_sync(0xffffffffu, !active || digit == d0)) {
        if ((threadIdx.x & 31) == lead) atomicAdd(&hist[d0], __popc(act));
        return;
    }
    if (active) atomicAdd(&hist[digit], 1);
}

// Warp 0: the digit whose bucket holds the need-th largest key of
// sh.hist[b] (counts by digit), the count above it and the bucket's size,
// into sh.digit[b], sh.above[b], sh.bucket[b].
template <int NT>
__device__ __forceinline__ void find_digit(SelectSharedT<NT> &sh, int b, int need)
{
    const int lane = threadIdx.x & 31;
    // lane l owns bins 255-8l .. 248-8l (descending)
    int c[8], tot = 0;
#pragma unroll
    for (int q = 0; q < 8; q++) {
        c[q] = sh.hist[b][255 - 8 * lane - q];
        tot += c[q];
    }
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    const int excl = incl - tot;
    if (excl < need && need <= incl) {
        int cum = excl;
#pragma unroll
        for (int q = 0; q < 8; q++) {
            if (cum + c[q] >= need) {
                sh.digit[b] = 255 - 8 * lane - q;
                sh.above[b] = cum;
                sh.bucket[b] = c[q];
                break;
            }
            cum += c[q];
        }
    }
}

// Radix select over n unique keys in shared memory: returns (prefix, mask)
// such that exactly `need` keys satisfy (key & mask) >= prefix.
// Requires 0 < need < n.  All threads of the CTA must call it.
template <int NT>
__device__ void radix_select(const uint64_t *keys, int n, int need, SelectSharedT<NT> &sh,
                             uint64_t &prefix_out, uint64_t &mask_out)
{
    // two barriers per pass: the counts and the result of a pass live in
    // one half of the double buffers while the other half, read by warp 0
    // one pass earlier, is zeroed for the next pass
    const int tid = threadIdx.x, warp = tid >> 5;
    uint64_t prefix = 0, mask = 0;
    for (int d = tid; d < 256; d += NT) sh.hist[0][d] = 0;
    __syncthreads();
    for (int shift = 56, cur = 0; shift >= 0; shift -= 8, cur ^= 1) {
        for (int d = tid; d < 256; d += NT) sh.hist[cur ^ 1][d] = 0;
        for (int base = 0; base < n; base += NT) {
            const int e = base + tid;
            const uint64_t k = e < n ? keys[e] : 0;
            hist_add(sh.hist[cur], e < n && (k & mask) == prefix, (int)((k >> shift) & 0xFF));
        }
        __syncthreads();
        if (warp == 0) find_digit(sh, cur, need);
        __syncthreads();
        need -= sh.above[cur];
        prefix |= (uint64_t)sh.digit[cur] << shift;
        mask |= (uint64_t)0xFF << shift;
        if (sh.bucket[cur] == need) break;   // the same decision in every thread
    }
    prefix_out = prefix;
    mask_out = mask;
}

// Exclusive CTA-wide prefix sum of one int per thread; also returns the total.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, SelectSharedT<NT> &sh, int &total)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += u;
    }
    if (lane == 31) sh.warp_tot[warp] = incl;
    __syncthreads();
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; w++) {
        const int x = sh.warp_tot[w];
        if (w < warp) base += x;
        tot += x;
    }
    __syncthreads();
    total = tot;
    return base + incl - v;
}

// Select the top `need` of n keys (already in ascending block order) and
// emit them in that order: to `final_row` as block ids between the forced
// entries (0 first, then the chosen, then D), or to `part` as keys.
template <int NT>
__device__ void select_and_emit(const uint64_t *keys, int n, int need, SelectSharedT<NT> &sh,
                                int32_t *final_row, int D, int topk, uint64_t *part)
{
    uint64_t prefix = 0, mask = 0;
    bool all = need >= n;
    if (need > 0 && !all) radix_select(keys, n, need, sh, prefix, mask);
    const int per = (n + NT - 1) / NT;
    const int e0 = threadIdx.x * per;
    const int e1 = min(e0 + per, n);
    int cnt = 0;
    if (need > 0)
        for (int e = e0; e < e1; e++) cnt += (all || (keys[e] & mask) >= prefix) ? 1 : 0;
    int total;
    int pos = block_exclusive_scan(cnt, sh, total);
    if (need > 0) {
        for (int e = e0; e < e1; e++) {
            const uint64_t k = keys[e];
            if (all || (k & mask) >= prefix) {
                if (final_row) final_row[1 + pos] = key_block(k);
                else part[pos] = k;
                pos++;
            }
        }
    }
    if (final_row) {
        const int chosen = need > 0 ? min(need, n) : 0;
        for (int s = threadIdx.x; s < topk; s += NT) {
            if (s == 0) final_row[0] = 0;
            else if (s == chosen + 1 && D > 0) final_row[s] = D;
            else if (s > chosen + (D > 0 ? 1 : 0)) final_row[s] = -1;
        }
    }
}

// ------------------------------------------ warp-level top-64 lists
// Per-token rows select from short chunks (a few hundred candidates per
// CTA), where the radix passes' barriers dominate.  There each warp sorts 64
// keys in registers with a bitonic network (element e = 32 r + lane in
// register r: a for r = 0, b for r = 1; 21 compare-exchange stages, strides
// below 32 through shuffles), and two sorted lists are cut to the top 64 of
// their union by one elementwise maximum against the other list reversed,
// which leaves a bitonic sequence, and a 6-stage bitonic merge.  Keys are
// unique, so every list is the exact top 64 by key; padding is key 0, below
// every candidate's key.
__device__ __forceinline__ uint64_t max64(uint64_t x, uint64_t y) { return x > y ? x : y; }
__device__ __forceinline__ uint64_t min64(uint64_t x, uint64_t y) { return x < y ? x : y; }

// One stage (block size k, stride j < 32) of a descending bitonic network
// (K: 64-bit selection keys, or 32-bit keys where they suffice -- half the
// shuffles).
template <typename K>
__device__ __forceinline__ void bitonic_stage(K &a, K &b, int k, int j)
{
    const int lane = threadIdx.x & 31;
    const K pa = __shfl_xor_sync(0xffffffffu, a, j);
    const K pb = __shfl_xor_sync(0xffffffffu, b, j);
    const bool lower = (lane & j) == 0;
    // the lower element of a pair keeps the maximum in a descending block
    const bool max_a = lower == ((lane & k) == 0);
    const bool max_b = lower == (((32 + lane) & k) == 0);
    a = max_a ? (a > pa ? a : pa) : (a < pa ? a : pa);
    b = max_b ? (b > pb ? b : pb) : (b < pb ? b : pb);
}

// Sorts the warp's 64 keys descending.
template <typename K>
__device__ __forceinline__ void warp_sort64_desc(K &a, K &b)
{
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) bitonic_stage(a, b, k, j);
    }
    // k = 64: the whole list descending
    const K hi = a > b ? a : b, lo = a < b ? a : b;
    a = hi;
    b = lo;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) bitonic_stage(a, b, 64, j);
}

// A bitonic sequence of 64 keys -> descending.
__device__ __forceinline__ void warp_merge64_desc(uint64_t &a, uint64_t &b)
{
    const uint64_t hi = max64(a, b), lo = min64(a, b);
    a = hi;
    b = lo;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) bitonic_stage(a, b, 64, j);
}

// (a, b) := the top 64 of the union of two descending lists (a, b) and
// (x, y), descending.
__device__ __forceinline__ void warp_top64_union(uint64_t &a, uint64_t &b, uint64_t x, uint64_t y)
{
    const int lane = threadIdx.x & 31;
    // element e of the other list reversed is its element 63 - e
    a = max64(a, __shfl_sync(0xffffffffu, y, 31 - lane));
    b = max64(b, __shfl_sync(0xffffffffu, x, 31 - lane));
    warp_merge64_desc(a, b);
}

// Top 64 (descending, padded with 0) of the n keys keys[0..n): each warp
// folds batches of 64 into a running list (a batch with no key above the
// list's 64th is skipped), then the warps' lists meet in a tree through
// `scratch` (8 x 64 keys), one block barrier per level.  The result is in
// warp 0's registers.  Every thread of the CTA calls it.
__device__ void cta_top64(const uint64_t *keys, int n, uint64_t *scratch, uint64_t &a_out, uint64_t &b_out)
{
    constexpr int NW = kSelThreads / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nbatch = (n + 63) / 64;
    const int nl = min(nbatch, NW);       // warps that hold a list
    uint64_t a = 0, b = 0;
    if (warp < nl) {
        bool first = true;
        for (int bt = warp; bt < nbatch; bt += NW) {
            const int e0 = bt * 64;
            uint64_t x = e0 + lane < n ? keys[e0 + lane] : 0;
            uint64_t y = e0 + 32 + lane < n ? keys[e0 + 32 + lane] : 0;
            if (!first) {
                const uint64_t thr = __shfl_sync(0xffffffffu, b, 31);
                if (!__any_sync(0xffffffffu, x > thr || y > thr)) continue;
            }
            warp_sort64_desc(x, y);
            if (first) {
                a = x;
                b = y;
                first = false;
            } else {
                warp_top64_union(a, b, x, y);
            }
        }
    }
    for (int step = 1; step < nl; step <<= 1) {
        // writers of this level and readers of the previous one use
        // different slots, so one barrier per level suffices
        if (warp < nl && (warp & (2 * step - 1)) == step) {
            scratch[warp * 64 + lane] = a;
            scratch[warp * 64 + 32 + lane] = b;
        }
        __syncthreads();
        if ((warp & (2 * step - 1)) == 0 && warp + step < nl) {
            const uint64_t *y = scratch + (warp + step) * 64;
            a = max64(a, y[63 - lane]);
            b = max64(b, y[31 - lane]);
            warp_merge64_desc(a, b);
        }
    }
    a_out = a;
    b_out = b;
}

// Warp 0 (holding the row's top-64 keys, descending): writes the row's
// indices -- 0, the m best candidates in ascending block order, D (if
// D > 0), then -1 -- by sorting the m block ids ascending in registers.
__device__ __forceinline__ void warp_emit_row(uint64_t a, uint64_t b, int m, int32_t *row, int D, int topk)
{
    const int lane = threadIdx.x & 31;
    // ascending ids = descending complements (32-bit keys: a candidate's id
    // is at least 1, so its complement is above the unused slots' 0)
    uint32_t x = lane < m ? 0xFFFFFFFFu - (uint32_t)key_block(a) : 0u;
    uint32_t y = 32 + lane < m ? 0xFFFFFFFFu - (uint32_t)key_block(b) : 0u;
    warp_sort64_desc(x, y);
    if (lane < m) row[1 + lane] = (int)(0xFFFFFFFFu - (uint32_t)x);
    if (32 + lane < m) row[33 + lane] = (int)(0xFFFFFFFFu - (uint32_t)y);
    for (int s = lane; s < topk; s += 32) {
        if (s == 0) row[0] = 0;
        else if (s == m + 1 && D > 0) row[s] = D;
        else if (s > m + (D > 0 ? 1 : 0)) row[s] = -1;
    }
}

// First query position of sequence b: q_pos0, or q_pos[b] for a ragged
// batch (device data, checked: a multiple of 64, at most q_pos0 -- the
// launch is planned for that furthest position -- and with the chunk of Tq
// tokens inside the summaries' capacity; otherwise QSA_ERR_BOUNDS and
// position 0).
__device__ __forceinline__ int seq_q_pos(const int32_t *q_pos, int b, int q_pos0, int Tq, int nblk_max,
                                         bool reporter)
{
    if (!q_pos) return q_pos0;
    const int qp = __ldg(q_pos + b);
    if (qp < 0 || (qp & 63) || qp > q_pos0 || (long)qp + Tq > 64L * nblk_max) {
        if (reporter) report(QSA_ERR_BOUNDS, 10);
        return 0;
    }
    return qp;
}

struct RowGeom {
    int D, ncand, m, nchunks;
};

__device__ __forceinline__ RowGeom row_geom(int i, int Tq, int q_pos0, int qblk, int topk, int CH)
{
    RowGeom g;
    const int t_last = min((i + 1) * qblk, Tq) - 1;
    g.D = (q_pos0 + t_last) / 64;
    g.ncand = max(g.D - 1, 0);
    const int nforced = g.D > 0 ? 2 : 1;
    g.m = min(topk - nforced, g.ncand);
    g.nchunks = max(1, (g.ncand + CH - 1) / CH);
    return g;
}

// V consecutive summary components as fp32: fp32 summaries as they are,
// bf16 summaries widened exactly (the scoring arithmetic is fp32 either way).
template <int V>
__device__ __forceinline__ void load_summary(const float *p, float (&k)[V])
{
    if constexpr (V == 4) {
        const float4 k4 = __ldg(reinterpret_cast<const float4 *>(p));
        k[0] = k4.x, k[1] = k4.y, k[2] = k4.z, k[3] = k4.w;
    } else {
        const float2 k2 = __ldg(reinterpret_cast<const float2 *>(p));
        k[0] = k2.x, k[1] = k2.y;
    }
}

template <int V>
__device__ __forceinline__ void load_summary(const __nv_bfloat16 *p, float (&k)[V])
{
    if constexpr (V == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        k[0] = __uint_as_float(u.x << 16), k[1] = __uint_as_float(u.x & 0xFFFF0000u);
        k[2] = __uint_as_float(u.y << 16), k[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
        const uint32_t u = __ldg(reinterpret_cast<const unsigned int *>(p));
        k[0] = __uint_as_float(u << 16), k[1] = __uint_as_float(u & 0xFFFF0000u);
    }
}

// Sums over the warp of 8 per-lane partials s[0..8) at once: a transposing
// butterfly that leaves the total of partial (lane >> 2) in the lanes with
// (lane & 3) == 0 (returned there).
__device__ __forceinline__ float reduce8(float (&s)[8])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int c = 0; c < 4; c++) {
        const bool up = lane & 16;
        const float send = up ? s[c] : s[c + 4];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
        s[c] = (up ? s[c + 4] : s[c]) + recv;
    }
#pragma unroll
    for (int c = 0; c < 2; c++) {
        const bool up = lane & 8;
        const float send = up ? s[c] : s[c + 2];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
        s[c] = (up ? s[c + 2] : s[c]) + recv;
    }
    {
        const bool up = lane & 4;
        const float send = up ? s[0] : s[1];
        const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
        s[0] = (up ? s[1] : s[0]) + recv;
    }
    s[0] += __shfl_xor_sync(0xffffffffu, s[0], 2);
    s[0] += __shfl_xor_sync(0xffffffffu, s[0], 1);
    return s[0];
}

// fp32 scores of n candidates (block summaries kc[0..n) of d = D fp32 or
// bf16 components, block ids j0..j0+n-1) against the pooled query qb, as
// 64-bit keys.  Each warp takes 8 candidates at a time; lane owns columns
// [lane*V, lane*V+V); a transposing butterfly leaves candidate (lane >> 2)
// of the group in lanes with (lane & 3) == 0.
template <int D, typename KcT>
__device__ __forceinline__ void score_chunk(const float *qb, const KcT *__restrict__ kc, int n, int j0,
                                            float sm_scale, uint64_t *keys)
{
    constexpr int V = D / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float q[V];
#pragma unroll
    for (int v = 0; v < V; v++) q[v] = qb[lane * V + v];
    const KcT *kc_base = kc + lane * V;
    for (int base = warp * 8; base < n; base += 8 * (kSelThreads / 32)) {
        float s[8];
#pragma unroll
        for (int c = 0; c < 8; c++) {
            s[c] = 0.f;
            if (base + c < n) {
                float k[V];
                load_summary<V>(kc_base + (long)(base + c) * D, k);
                if constexpr (V == 4) s[c] = q[0] * k[0] + q[1] * k[1] + q[2] * k[2] + q[3] * k[3];
                else s[c] = q[0] * k[0] + q[1] * k[1];
            }
        }
        const float dot = reduce8(s);
        const int e = base + (lane >> 2);
        if ((lane & 3) == 0 && e < n) keys[e] = make_key(dot * sm_scale, j0 + e);
    }
}

// Per-token rows: this lane's columns [lane*V, lane*V+V) of the pooled query
// -- the fp32 sum over the token's G head rows (qt: the group's first head),
// in head order, times 1/G -- in registers, so that no block barrier stands
// between the query's loads and the first summary loads.
template <int D>
__device__ __forceinline__ void pooled_query_lane(const __nv_bfloat16 *__restrict__ qt, int G, float (&q)[D / 32])
{
    constexpr int V = D / 32;
    const int lane = threadIdx.x & 31;
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; v++) acc[v] = 0.f;
    for (int h = 0; h < G; h++) {
        float x[V];
        load_summary<V>(qt + (long)h * D + lane * V, x);   // bf16 widened exactly
#pragma unroll
        for (int v = 0; v < V; v++) acc[v] += x[v];
    }
    const float inv = 1.0f / (float)G;
#pragma unroll
    for (int v = 0; v < V; v++) q[v] = acc[v] * inv;
}

// score_chunk with the pooled query in registers (pooled_query_lane).
template <int D, typename KcT>
__device__ __forceinline__ void score_chunk_q(const float (&q)[D / 32], const KcT *__restrict__ kc, int n, int j0,
                                              float sm_scale, uint64_t *keys)
{
    constexpr int V = D / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const KcT *kc_base = kc + lane * V;
    for (int base = warp * 8; base < n; base += 8 * (kSelThreads / 32)) {
        float s[8];
#pragma unroll
        for (int c = 0; c < 8; c++) {
            s[c] = 0.f;
            if (base + c < n) {
                float k[V];
                load_summary<V>(kc_base + (long)(base + c) * D, k);
                if constexpr (V == 4) s[c] = q[0] * k[0] + q[1] * k[1] + q[2] * k[2] + q[3] * k[3];
                else s[c] = q[0] * k[0] + q[1] * k[1];
            }
        }
        const float dot = reduce8(s);
        const int e = base + (lane >> 2);
        if ((lane & 3) == 0 && e < n) keys[e] = make_key(dot * sm_scale, j0 + e);
    }
}

// Per-head logits of n blocks (summaries kc[0..n)) for the G <= 8 heads of
// a group (queries qh[h][0..D), fp32): for every block e, f(e, z) receives
// z[h] = scale * <qh[h], kc[e]> for h < G, in the lane that holds them
// ((lane & 3) == 0).  Each warp takes 8 blocks at a time and loads each
// summary once for all heads.
template <int D, typename KcT, typename F>
__device__ __forceinline__ void head_logits(const float (*qh)[D], int G, const KcT *__restrict__ kc, int n,
                                            float scale, F &&f)
{
    constexpr int V = D / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const KcT *kc_base = kc + lane * V;
    for (int base = warp * 8; base < n; base += 8 * (kSelThreads / 32)) {
        float k[8][V];
#pragma unroll
        for (int c = 0; c < 8; c++) {
            if (base + c < n) {
                load_summary<V>(kc_base + (long)(base + c) * D, k[c]);
            } else {
#pragma unroll
                for (int v = 0; v < V; v++) k[c][v] = 0.f;
            }
        }
        float z[8];
#pragma unroll
        for (int h = 0; h < 8; h++) {
            z[h] = 0.f;
            if (h < G) {
                float s[8];
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    s[c] = 0.f;
#pragma unroll
                    for (int v = 0; v < V; v++) s[c] += qh[h][lane * V + v] * k[c][v];
                }
                z[h] = reduce8(s) * scale;
            }
        }
        const int e = base + (lane >> 2);
        if ((lane & 3) == 0 && e < n) f(e, z);
    }
}

// Longest chunk whose softmax-sum logits (8 heads) stay in shared memory.
constexpr int kSoftmaxZCap = 1024;

// Running (max, sum of 2^(z - max)) pairs, merged; an empty pair is
// (-inf, 0).
__device__ __forceinline__ void lse2_merge(float &m, float &s, float m2, float s2)
{
    const float mn = fmaxf(m, m2);
    if (mn == -INFINITY) return;   // both empty
    s = s * fast_exp2(m - mn) + s2 * fast_exp2(m2 - mn);
    m = mn;
}

// --------------------------------------------------------- score+select
// grid (maxchunks, NR, B*Hkv); dynamic smem CH * 8 bytes.
// FROM_SCORES: the candidates' scores come from a table [B*Hkv][NR][nblk_max]
// written by another scoring kernel (the aggregator variants) instead of
// the pooled-query dots.
template <int D, typename KcT, bool FROM_SCORES = false, int NT = kSelThreads>
__global__ void __launch_bounds__(NT) score_select_kernel(
    const float *__restrict__ Qbar, const KcT *__restrict__ Kc, int32_t *__restrict__ idx,
    uint64_t *__restrict__ part, int nblk_max, int Tq, int q_pos0, int qblk, int topk,
    float sm_scale, int CH, int maxchunks, int Hkv, const int32_t *__restrict__ q_pos,
    const float *__restrict__ scores = nullptr, int score_stride = 0)
{
    static_assert(FROM_SCORES || NT == kSelThreads, "the scoring path is written for kSelThreads threads");
    extern __shared__ uint64_t keys[];
    __shared__ SelectSharedT<NT> sh;
    const int chunk = blockIdx.x, i = blockIdx.y, bg = blockIdx.z, NR = gridDim.y;
    const int qp = seq_q_pos(q_pos, bg / Hkv, q_pos0, Tq, nblk_max,
                             threadIdx.x == 0 && chunk == 0 && i == 0 && bg % Hkv == 0);
    const RowGeom g = row_geom(i, Tq, qp, qblk, topk, CH);
    if (chunk >= g.nchunks) return;
    const int j0 = 1 + chunk * CH;
    const int n = max(0, min(CH, g.ncand - chunk * CH));
    const long row = (long)bg * NR + i;

    if constexpr (FROM_SCORES) {
        const float *srow = scores + row * (score_stride ? score_stride : nblk_max) + j0;
        // eight loads in flight per thread before their keys are stored
        for (int e0 = threadIdx.x; e0 < n; e0 += 8 * NT) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) v[u] = e0 + u * NT < n ? __ldg(srow + e0 + u * NT) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; u++)
                if (e0 + u * NT < n) keys[e0 + u * NT] = make_key(v[u], j0 + e0 + u * NT);
        }
    } else {
        score_chunk<D, KcT>(Qbar + row * D, Kc + ((long)bg * nblk_max + j0) * D, n, j0, sm_scale, keys);
    }
    __syncthreads();

    const int need = min(g.m, n);
    if (g.nchunks == 1) {
        select_and_emit(keys, n, need, sh, idx + row * topk, g.D, topk, nullptr);
    } else {
        select_and_emit(keys, n, need, sh, nullptr, g.D, topk,
                        part + (row * maxchunks + chunk) * kMaxChosen);
    }
}

// ---------------------------------------------- prefill rows: score table
// Consecutive prefill rows of one (b, g) share almost all their candidates
// (row i's are blocks 1 .. D_i - 1), so the scores of a 64-row x 64-candidate
// tile are an fp32 matrix product Qbar_tile (64 x D) * Kc_tile^T (D x 64)
// over shared memory: every summary and pooled query crosses L2 once per
// tile instead of once per row.  One CTA per tile; the tiles go to shared
// memory by cp.async (fp32; bf16 summaries are widened on the way).  Each
// thread forms a 4 x 4 block of dots (rows 4 ty .. 4 ty + 3, candidates tx,
// tx + 16, tx + 32, tx + 48) with fp32 FMAs in increasing d; rows are padded
// to D + 4 floats so the 16-byte shared loads of the 16 candidate columns a
// warp reads fall in distinct banks.  The scores go into a table
// [B*Hkv][NR][stride] that score_select_kernel<.., true> selects from;
// tiles wholly past their rows' diagonals are skipped.
// Sharded caches: the candidates are restricted to blocks [lo, hi) (lo >= 1),
// Kc holds the summaries of blocks kc_lo .. kc_lo + kc_n - 1 of each (b, g)
// (the rank's own range), and table column c is block tab_lo + c.  The
// whole cache: lo = 1, hi = INT_MAX, kc_lo = 0, kc_n = T_kv_max / 64,
// tab_lo = 0 (column = block index).
// grid (ceil(max candidates / 64), ceil(NR / 64), B*Hkv); 256 threads;
// dynamic shared memory 2 * 64 * (D + 4) * 4 bytes.
constexpr int kTableTile = 64;

template <int D, typename KcT>
__global__ void __launch_bounds__(256) score_table_kernel(
    const float *__restrict__ Qbar, const KcT *__restrict__ Kc, float *__restrict__ table, int nblk_max, int Tq,
    int q_pos0, int stride, float sm_scale, int Hkv, const int32_t *__restrict__ q_pos, int lo, int hi, int kc_lo,
    int kc_n, int tab_lo)
{
    constexpr int T = kTableTile, LD = D + 4, CPR = D / 4;   // CPR: 16-byte chunks (of fp32) per row
    extern __shared__ __align__(16) float tsm[];
    float *qs = tsm;                  // [T][LD] pooled queries of the tile's rows
    float *ks = tsm + T * LD;         // [T][LD] summaries of the tile's candidates
    const int bg = blockIdx.z, NR = (Tq + 63) / 64;
    const int qp = seq_q_pos(q_pos, bg / Hkv, q_pos0, Tq, nblk_max, false);
    const int r0 = blockIdx.y * T, nr = min(T, NR - r0);
    // candidates of the CTA that some row of its tile has (j < D of the last row)
    const int Dlast = (qp + min((r0 + nr) * 64, Tq) - 1) / 64;
    const int j0 = lo + blockIdx.x * T;
    const int jend = min(min(Dlast, hi), j0 + T);
    if (jend <= j0) return;
    const int tid = threadIdx.x;
    // summaries of candidates j0 .. j0 + T - 1 (zero past jend)
    {
        for (int e = tid; e < T * CPR; e += 256) {
            const int rr = e / CPR, c = e % CPR;
            const bool valid = j0 + rr < jend;
            const KcT *src = Kc + ((long)bg * kc_n + (valid ? j0 + rr - kc_lo : 0)) * D + 4 * c;
            if constexpr (sizeof(KcT) == 4) {
                cp_async16(ks + rr * LD + 4 * c, src, valid);
            } else {
                float k4[4] = {0.f, 0.f, 0.f, 0.f};
                if (valid) load_summary<4>(src, k4);
                *reinterpret_cast<float4 *>(ks + rr * LD + 4 * c) = make_float4(k4[0], k4[1], k4[2], k4[3]);
            }
        }
    }
    for (int e = tid; e < T * CPR; e += 256) {
        const int rr = e / CPR, c = e % CPR;
        const bool valid = rr < nr;
        cp_async16(qs + rr * LD + 4 * c, Qbar + ((long)bg * NR + r0 + (valid ? rr : 0)) * D + 4 * c, valid);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    const int ty = tid >> 4, tx = tid & 15;
    {
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; i++)
#pragma unroll
            for (int jj = 0; jj < 4; jj++) acc[i][jj] = 0.f;
        const float *qrow = qs + (4 * ty) * LD;
        const float *krow = ks + tx * LD;
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
            float4 a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; i++) a[i] = *reinterpret_cast<const float4 *>(qrow + i * LD + d);
#pragma unroll
            for (int jj = 0; jj < 4; jj++) b[jj] = *reinterpret_cast<const float4 *>(krow + 16 * jj * LD + d);
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int jj = 0; jj < 4; jj++) {
                    acc[i][jj] = fmaf(a[i].x, b[jj].x, acc[i][jj]);
                    acc[i][jj] = fmaf(a[i].y, b[jj].y, acc[i][jj]);
                    acc[i][jj] = fmaf(a[i].z, b[jj].z, acc[i][jj]);
                    acc[i][jj] = fmaf(a[i].w, b[jj].w, acc[i][jj]);
                }
        }
        const int nc = min(T, jend - j0);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int rr = 4 * ty + i;
            if (rr >= nr) break;
            const int Drow = (qp + min((r0 + rr + 1) * 64, Tq) - 1) / 64;
            float *trow = table + ((long)bg * NR + r0 + rr) * stride + (j0 - tab_lo);
#pragma unroll
            for (int jj = 0; jj < 4; jj++) {
                const int e = tx + 16 * jj;
                if (e < nc && j0 + e < Drow) trow[e] = acc[i][jj] * sm_scale;
            }
        }
    }
}

// grid (NR, B*Hkv); dynamic smem maxchunks * kMaxChosen * 8 bytes.
__global__ void __launch_bounds__(kSelThreads) merge_select_kernel(
    const uint64_t *__restrict__ part, int32_t *__restrict__ idx, int Tq, int q_pos0, int qblk,
    int topk, int CH, int maxchunks, int Hkv, int nblk_max, const int32_t *__restrict__ q_pos)
{
    extern __shared__ uint64_t keys[];
    __shared__ SelectShared sh;
    const int i = blockIdx.x, bg = blockIdx.y, NR = gridDim.x;
    const int qp = seq_q_pos(q_pos, bg / Hkv, q_pos0, Tq, nblk_max, false);
    const RowGeom g = row_geom(i, Tq, qp, qblk, topk, CH);
    if (g.nchunks <= 1) return;
    const long row = (long)bg * NR + i;
    // concatenate the chunks' lists (each ascending, chunks ascending)
    int n = 0;
    for (int c = 0; c < g.nchunks; c++) {
        const int nc = min(g.m, min(CH, g.ncand - c * CH));
        const uint64_t *src = part + (row * maxchunks + c) * kMaxChosen;
        for (int e = threadIdx.x; e < nc; e += kSelThreads) keys[n + e] = src[e];
        n += nc;
    }
    __syncthreads();
    select_and_emit(keys, n, g.m, sh, idx + row * topk, g.D, topk, nullptr);
}

// ---------------------------------------------------- sharded caches
// A rank that owns the cache blocks [lo, hi) selects, for every prefill row,
// the top m of its own candidates (blocks j in [lo, hi) with 1 <= j < D) in
// chunks of CH from the score table (column j - lo), and writes each
// chunk's keys, in block order, as a list of kMaxChosen keys padded with 0
// (below every candidate's key): part[row][chunk][kMaxChosen].  The lists
// of all ranks, gathered, hold the row's top m (a candidate outside a
// list's top m has m better ones in the same list), and merge_lists_kernel
// picks it from them.
// grid (maxchunks, NR, B*Hkv); dynamic smem CH * 8 bytes.
__global__ void __launch_bounds__(kSelThreads) local_lists_kernel(
    const float *__restrict__ table, uint64_t *__restrict__ part, int nblk_max, int Tq, int q_pos0, int topk, int CH,
    int maxchunks, int Hkv, int lo, int hi, int stride)
{
    extern __shared__ uint64_t keys[];
    __shared__ SelectShared sh;
    const int chunk = blockIdx.x, i = blockIdx.y, bg = blockIdx.z, NR = gridDim.y;
    const RowGeom g = row_geom(i, Tq, q_pos0, 64, topk, CH);
    const int first = max(1, lo), last = min(g.D - 1, hi - 1);   // the row's own candidates
    const int j0 = first + chunk * CH;
    const int n = max(0, min(CH, last - j0 + 1));
    const long row = (long)bg * NR + i;
    uint64_t *dst = part + (row * maxchunks + chunk) * kMaxChosen;
    const float *srow = table + row * stride + (j0 - lo);
    for (int e = threadIdx.x; e < n; e += kSelThreads) keys[e] = make_key(__ldg(srow + e), j0 + e);
    __syncthreads();
    const int need = min(g.m, n);
    select_and_emit(keys, n, need, sh, nullptr, g.D, topk, dst);
    for (int e = max(need, 0) + threadIdx.x; e < kMaxChosen; e += kSelThreads) dst[e] = 0;
}

// The row's selection from the ranks' lists as an all-gather leaves them
// (rank-major: lists[r][row][nlists][kMaxChosen], 0 = padding), taken in
// rank order -- ascending block ranges, each rank's chunks in order -- so
// the keys stand in ascending block order: the top m by key, then the
// forced blocks.
// grid (NR, B*Hkv); dynamic smem nranks * nlists * kMaxChosen * 8 bytes.
__global__ void __launch_bounds__(kSelThreads) merge_lists_kernel(
    const uint64_t *__restrict__ lists, int32_t *__restrict__ idx, int Tq, int q_pos0, int topk, int nlists,
    int nranks)
{
    extern __shared__ uint64_t keys[];
    __shared__ SelectShared sh;
    const int i = blockIdx.x, bg = blockIdx.y, NR = gridDim.x;
    const RowGeom g = row_geom(i, Tq, q_pos0, 64, topk, 1 << 30);
    const long row = (long)bg * NR + i, rows = (long)gridDim.y * NR;
    const int per = nlists * kMaxChosen, n = nranks * per;
    for (int e = threadIdx.x; e < n; e += kSelThreads) keys[e] = lists[((long)(e / per) * rows + row) * per + e % per];
    __syncthreads();
    select_and_emit(keys, n, g.m, sh, idx + row * topk, g.D, topk, nullptr);
}

// Partial attention outputs of the ranks (each over its own blocks, with its
// natural-log normaliser lse_r; lse_r = -inf when it owns none of the row's
// blocks) merged into the row's output: O = sum_r exp(lse_r - L) O_r with
// L = log sum_r exp(lse_r), and lse = L.  D/8 lanes per (token, head) row,
// each owning 8 consecutive columns (one 16-byte load per rank; the first
// 8 ranks' loads all in flight before any arithmetic); the ranks are added
// in ascending order, in fp32.  grid ceil(rows / (8 * 256 / D)); 256 threads.
template <int D>
__global__ void __launch_bounds__(256) merge_partials_kernel(const __nv_bfloat16 *__restrict__ O_parts,
                                                             const float *__restrict__ lse_parts,
                                                             __nv_bfloat16 *__restrict__ O, float *__restrict__ lse,
                                                             int nparts, long rows)
{
    // a lane owns 8 columns (one 16-byte load per rank); D / 8 lanes per row
    constexpr int LPR = D / 8, RPW = 32 / LPR;
    const int lane = threadIdx.x & 31, cl = lane % LPR;
    const long row = ((long)blockIdx.x * 8 + (threadIdx.x >> 5)) * RPW + lane / LPR;
    if (row >= rows) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(O_parts + row * D) + cl;
    const long rstride = rows * (D / 8);   // uint4 per rank
    // the first (up to) 8 ranks' normalisers and columns all in flight at once
    constexpr int RF = 8;
    const int nf = min(nparts, RF);
    float l[RF];
    uint4 v[RF];
#pragma unroll
    for (int r = 0; r < RF; r++)
        if (r < nf) {
            l[r] = __ldg(lse_parts + (long)r * rows + row);
            v[r] = __ldg(src + r * rstride);
        }
    float m = -INFINITY;
#pragma unroll
    for (int r = 0; r < RF; r++)
        if (r < nf) m = fmaxf(m, l[r]);
    for (int r = RF; r < nparts; r++) m = fmaxf(m, __ldg(lse_parts + (long)r * rows + row));
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; c++) acc[c] = 0.f;
    float wsum = 0.f;
    // ranks in ascending order
    auto add = [&](float lr, const uint4 &vr) {
        const float w = __expf(lr - m);
        wsum += w;
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&vr);
#pragma unroll
        for (int c = 0; c < 4; c++) {
            const float2 f = __bfloat1622float2(h[c]);
            acc[2 * c] += w * f.x;
            acc[2 * c + 1] += w * f.y;
        }
    };
    if (m != -INFINITY) {
#pragma unroll
        for (int r = 0; r < RF; r++)
            if (r < nf) add(l[r], v[r]);
        for (int r = RF; r < nparts; r++) add(__ldg(lse_parts + (long)r * rows + row), __ldg(src + r * rstride));
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint4 out;
    __nv_bfloat162 *oh = reinterpret_cast<__nv_bfloat162 *>(&out);
#pragma unroll
    for (int c = 0; c < 4; c++) oh[c] = __floats2bfloat162_rn(acc[2 * c] * inv, acc[2 * c + 1] * inv);
    reinterpret_cast<uint4 *>(O + row * D)[cl] = out;
    if (lse && cl == 0) lse[row] = m == -INFINITY ? -INFINITY : m + __logf(wsum);
}

// ------------------------------------------------ per-token, one launch
// grid (NCH, Tq, B*Hkv) with cluster (NCH, 1, 1); dynamic shared memory
// CH * 8 bytes.  Row i = token i (qblk = 1).  Every CTA pools its token's
// query over the group's heads, scores its chunk of summaries and selects
// the chunk's top-m; it stores that list straight into the leader's shared
// memory (distributed-shared-memory stores, padded with key 0, which is
// below every score's key).  After one cluster barrier the other CTAs are
// done and the leader selects the row's top-m from the lists, which are in
// block order.
// Ragged batches: with seq_lens given (one decode token per sequence,
// Tq = 1), sequence b's token sits at position seq_lens[b] - 1 (checked
// against the summaries' capacity; an invalid length reports
// QSA_ERR_BOUNDS and the row keeps block 0 only).
template <int D, typename KcT, bool SOFTMAX>
__device__ __forceinline__ void select_token_body(
    const __nv_bfloat16 *__restrict__ Q, const KcT *__restrict__ Kc, int32_t *__restrict__ idx,
    int nblk_max, int Tq, int Hq, int Hkv, int q_pos0, int topk, float sm_scale, int CH,
    const int32_t *__restrict__ seq_lens)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ uint64_t keys[];                 // [CH] this chunk's keys
    __shared__ uint64_t scratch[8 * 64];               // the warps' top-64 lists meeting in a tree
    __shared__ uint64_t lists[8 * 64];                 // leader: the chunks' top-64 lists
    const int NCH = (int)cluster.num_blocks();
    const int chunk = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i = blockIdx.y, bg = blockIdx.z, NR = gridDim.y;
    const int b = bg / Hkv, grp = bg % Hkv, G = Hq / Hkv;
    const long row = (long)bg * NR + i;
    grid_dependency_wait();     // Q and Kc come from earlier work on the stream
    grid_launch_dependents();   // the attention that reads idx may be scheduled
    int qp = q_pos0;
    if (seq_lens) {
        qp = __ldg(seq_lens + b) - 1;
        if (qp < 0 || qp >= 64 * nblk_max) {
            if (tid == 0 && chunk == 0) report(QSA_ERR_BOUNDS, 8);
            qp = 0;
        }
    }
    const RowGeom g = row_geom(i, Tq, qp, 1, topk, CH);

    const int j0 = 1 + chunk * CH;
    const int n = max(0, min(CH, g.ncand - chunk * CH));
    if constexpr (SOFTMAX) {
        // Softmax-sum aggregator: s_j = sum over the group's heads h of
        // softmax over the blocks {0, ..., D-1} of z_h = sm_scale <q_h, Kc_j>,
        // at j.  Pass 1: each CTA's (max, sum) per head over its blocks
        // (chunk 0 also takes block 0, which is in the normalisation set but
        // not a candidate), merged across the cluster through distributed
        // shared memory; pass 2: the candidates' scores from the merged
        // statistics (the summaries are read again, mostly from L2).  Base-2
        // logits: the softmax is the same.
        __shared__ float qh[8][D];
        __shared__ float wst[kSelThreads / 32][8][2];
        __shared__ float cst[8][2];
        __shared__ float gst[8][2];
        const __nv_bfloat16 *qt = Q + (((long)b * Tq + i) * Hq + (long)grp * G) * D;
        for (int e = tid; e < G * D; e += kSelThreads) qh[e / D][e % D] = __bfloat162float(qt[e]);
        __syncthreads();
        const float scale = sm_scale * 1.4426950408889634f;
        if (g.ncand > 0) {
            const int js = chunk == 0 ? 0 : j0;
            const int ns = n + (j0 - js);
            // logits kept in shared memory after the keys when the chunk is
            // short enough (kSoftmaxZCap), else recomputed in pass 2
            const bool zsm = CH <= kSoftmaxZCap;
            float *zb = reinterpret_cast<float *>(keys + CH);   // [8][CH + 1]
            const int zs = CH + 1;
            if (zsm) {
                head_logits<D, KcT>(qh, G, Kc + ((long)bg * nblk_max + js) * D, ns, scale,
                                    [&](int e, const float(&z)[8]) {
#pragma unroll
                                        for (int h = 0; h < 8; h++)
                                            if (h < G) zb[h * zs + e] = z[h];
                                    });
                __syncthreads();
                if (warp < G) {   // warp h: head h's (max, sum) over this CTA's blocks
                    const float *zr = zb + warp * zs;
                    float m = -INFINITY;
                    for (int e = lane; e < ns; e += 32) m = fmaxf(m, zr[e]);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                    float sum = 0.f;
                    if (m != -INFINITY)
                        for (int e = lane; e < ns; e += 32) sum += fast_exp2(zr[e] - m);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                    if (lane == 0) cst[warp][0] = m, cst[warp][1] = sum;
                }
            } else {
                float mr[8], sr[8];
#pragma unroll
                for (int h = 0; h < 8; h++) mr[h] = -INFINITY, sr[h] = 0.f;
                head_logits<D, KcT>(qh, G, Kc + ((long)bg * nblk_max + js) * D, ns, scale,
                                    [&](int, const float(&z)[8]) {
#pragma unroll
                                        for (int h = 0; h < 8; h++)
                                            if (h < G) lse2_merge(mr[h], sr[h], z[h], 1.f);
                                    });
#pragma unroll
                for (int h = 0; h < 8; h++) {
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float m2 = __shfl_xor_sync(0xffffffffu, mr[h], off);
                        const float s2 = __shfl_xor_sync(0xffffffffu, sr[h], off);
                        lse2_merge(mr[h], sr[h], m2, s2);
                    }
                    if (lane == 0) wst[warp][h][0] = mr[h], wst[warp][h][1] = sr[h];
                }
                __syncthreads();
                if (tid < G) {
                    float m = -INFINITY, sm = 0.f;
                    for (int w = 0; w < kSelThreads / 32; w++) lse2_merge(m, sm, wst[w][tid][0], wst[w][tid][1]);
                    cst[tid][0] = m, cst[tid][1] = sm;
                }
            }
            if (g.nchunks > 1) {
                cluster.sync();   // every CTA's statistics are in place
                if (tid < G) {
                    float m = -INFINITY, sm = 0.f;
                    for (int c = 0; c < NCH; c++) {
                        const float *r = &cluster.map_shared_rank(&cst[0][0], c)[2 * tid];
                        lse2_merge(m, sm, r[0], r[1]);
                    }
                    gst[tid][0] = m, gst[tid][1] = 1.f / sm;
                }
            } else {
                __syncthreads();
                if (tid < G) gst[tid][0] = cst[tid][0], gst[tid][1] = 1.f / cst[tid][1];
            }
            __syncthreads();
            if (zsm) {
                for (int e = tid; e < n; e += kSelThreads) {
                    float acc = 0.f;
#pragma unroll
                    for (int h = 0; h < 8; h++)
                        if (h < G) acc += fast_exp2(zb[h * zs + e + (j0 - js)] - gst[h][0]) * gst[h][1];
                    keys[e] = make_key(acc, j0 + e);
                }
            } else {
                head_logits<D, KcT>(qh, G, Kc + ((long)bg * nblk_max + j0) * D, n, scale,
                                    [&](int e, const float(&z)[8]) {
                                        float acc = 0.f;
#pragma unroll
                                        for (int h = 0; h < 8; h++)
                                            if (h < G) acc += fast_exp2(z[h] - gst[h][0]) * gst[h][1];
                                        keys[e] = make_key(acc, j0 + e);
                                    });
            }
        }
    } else {
        // pooled query: mean of the token's query over the group's heads
        float q[D / 32];
        pooled_query_lane<D>(Q + (((long)b * Tq + i) * Hq + (long)grp * G) * D, G, q);
        score_chunk_q<D, KcT>(q, Kc + ((long)bg * nblk_max + j0) * D, n, j0, sm_scale, keys);
    }
    __syncthreads();
    // the chunk's top 64 (the row keeps at most 62 candidates)
    uint64_t a, bk;
    cta_top64(keys, n, scratch, a, bk);
    if (g.nchunks == 1) {
        // chunk 0 holds every candidate of the row (the other CTAs only
        // scored nothing): emit directly, no cluster exchange
        if (chunk == 0 && warp == 0) warp_emit_row(a, bk, g.m, idx + row * topk, g.D, topk);
        return;
    }
    if (warp == 0) {
        // this chunk's list into the leader's shared memory
        uint64_t *dst = cluster.map_shared_rank(lists, 0) + chunk * 64;
        dst[lane] = a;
        dst[32 + lane] = bk;
    }
    cluster.sync();   // every list is in the leader
    if (chunk != 0) return;
    // the leader: the chunks' lists meet in a tree (warp c starts from list c)
    a = bk = 0;
    if (warp < NCH) {
        a = lists[warp * 64 + lane];
        bk = lists[warp * 64 + 32 + lane];
    }
    for (int step = 1; step < NCH; step <<= 1) {
        if (warp < NCH && (warp & (2 * step - 1)) == step) {
            scratch[warp * 64 + lane] = a;
            scratch[warp * 64 + 32 + lane] = bk;
        }
        __syncthreads();
        if ((warp & (2 * step - 1)) == 0 && warp + step < NCH) {
            const uint64_t *y = scratch + (warp + step) * 64;
            a = max64(a, y[63 - lane]);
            bk = max64(bk, y[31 - lane]);
            warp_merge64_desc(a, bk);
        }
    }
    if (warp == 0) warp_emit_row(a, bk, g.m, idx + row * topk, g.D, topk);
}

template <int D, typename KcT>
__global__ void __launch_bounds__(kSelThreads) select_token_kernel(
    const __nv_bfloat16 *__restrict__ Q, const KcT *__restrict__ Kc, int32_t *__restrict__ idx,
    int nblk_max, int Tq, int Hq, int Hkv, int q_pos0, int topk, float sm_scale, int CH,
    const int32_t *__restrict__ seq_lens)
{
    select_token_body<D, KcT, false>(Q, Kc, idx, nblk_max, Tq, Hq, Hkv, q_pos0, topk, sm_scale, CH, seq_lens);
}

// The softmax-sum aggregator's per-token selection: at most 64 registers,
// so that 4 CTAs share an SM and a decode batch's clusters run in one wave.
template <int D, typename KcT>
__global__ void __launch_bounds__(kSelThreads, 4) select_token_softmax_kernel(
    const __nv_bfloat16 *__restrict__ Q, const KcT *__restrict__ Kc, int32_t *__restrict__ idx,
    int nblk_max, int Tq, int Hq, int Hkv, int q_pos0, int topk, float sm_scale, int CH,
    const int32_t *__restrict__ seq_lens)
{
    select_token_body<D, KcT, true>(Q, Kc, idx, nblk_max, Tq, Hq, Hkv, q_pos0, topk, sm_scale, CH, seq_lens);
}

}  // namespace qsa
