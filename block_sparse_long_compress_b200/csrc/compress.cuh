// Step 1 -- key compression: the fp32 mean of the 64 keys of a block
// (pages "Qwen4 architecture: QSA, GR, PLE", section 1, "compress into
// small blocks"; "Qwen4 in llama.cpp: Dissecting PR #27742", section "QSA Is
// an Address-Selection Problem, Not a New Attention Equation",
// "compressed-block representation").
//
// HBM-bound: per block it reads 64*d bf16 and writes d fp32.  One CTA of
// 128 threads per (b, h, block); thread t owns the 16-byte column chunk
// t % (d/8) and the rows r = t / (d/8) + k*R (R = 128 / (d/8) row lanes),
// issuing all its loads before the first add.  The reduction order is fixed
// (each thread adds its rows in increasing r, then row lanes are added in
// increasing lane order), so results are bit-reproducible.  The summary is
// stored as fp32, or (the bf16-summary option) as that fp32 mean rounded to
// the nearest bf16, ties to even -- half the bytes for the scoring to read.
// Paged caches (serving): logical block j of sequence b is read from page
// block_table[b][j] of [num_pages][Hkv][64][d], and with seq_lens given only
// complete blocks (64 (j+1) <= seq_lens[b]) are written; summaries stay in
// logical order [B][Hkv][max_blocks][d].
#pragma once
#include "device.cuh"

namespace qsa {

__device__ __forceinline__ void store_summary(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_summary(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

template <int D, typename KcT>
__global__ void __launch_bounds__(128) compress_keys_kernel(const __nv_bfloat16 *__restrict__ K,
                                                            KcT *__restrict__ Kc, int T_kv_max,
                                                            int nblk_max, int blk_begin,
                                                            int nblk,
                                                            const int32_t *__restrict__ block_table,
                                                            const int32_t *__restrict__ seq_lens,
                                                            int Hkv, int num_pages)
{
    constexpr int CHUNKS = D / 8;            // 16-byte chunks per key row
    constexpr int LANES = 128 / CHUNKS;      // row lanes
    constexpr int ROWS = 64 / LANES;         // rows per thread
    __shared__ float part[LANES][D];

    const int j = blk_begin + (int)(blockIdx.x % (unsigned)nblk);
    const long bh = blockIdx.x / (unsigned)nblk;
    const int t = threadIdx.x;
    const int c = t % CHUNKS, lane = t / CHUNKS;

    long row0 = bh * T_kv_max + (long)j * 64;
    if (block_table) {
        const long b = bh / Hkv, h = bh % Hkv;
        if (seq_lens && 64L * (j + 1) > (long)__ldg(seq_lens + b)) return;   // incomplete: not yet
        const int page = __ldg(block_table + b * nblk_max + j);
        if (page < 0 || page >= num_pages) {
            if (threadIdx.x == 0) report(QSA_ERR_BOUNDS, 9);
            return;
        }
        row0 = ((long)page * Hkv + h) * 64;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(K + row0 * D);
    uint4 v[ROWS];
#pragma unroll
    for (int k = 0; k < ROWS; k++) v[k] = __ldg(src + (long)(lane + k * LANES) * CHUNKS + c);

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; e++) acc[e] = 0.f;
#pragma unroll
    for (int k = 0; k < ROWS; k++) {
        const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v[k]);
#pragma unroll
        for (int e = 0; e < 4; e++) {
            float2 f = __bfloat1622float2(p[e]);
            acc[2 * e] += f.x;
            acc[2 * e + 1] += f.y;
        }
    }
#pragma unroll
    for (int e = 0; e < 8; e++) part[lane][c * 8 + e] = acc[e];
    __syncthreads();
    if (t < D) {
        float s = 0.f;
#pragma unroll
        for (int l = 0; l < LANES; l++) s += part[l][t];
        store_summary(Kc + (bh * nblk_max + j) * D + t, s * (1.0f / 64.0f));
    }
}

}  // namespace qsa
