// Quantized-KV option for decode -- the rotated cache representation of
// page "Qwen4 in llama.cpp: Dissecting PR #27742", section "Quantized KV
// Exposed a Backend Storage Invariant": K and V are stored in a
// Walsh-Hadamard-rotated basis (spreading channel outliers before
// quantization), attention runs in that basis and the output is rotated
// back (H^2 = I for the normalised transform).
//
// Each cache row of d = 128 bf16 values x becomes u = WHT(x) (unnormalised,
// fp32), one fp32 scale s = max|u| / 448 and 128 fp8 e4m3 codes
// e4m3(u / s) (nearest, ties to even, saturating): u ~= s * code.  The
// normalised rotation is u / sqrt(128); the decode kernel folds the factor
// 1/128 that two of them make into the score scale and the back-rotation,
// so no irrational constant enters a code.  One warp per row; HBM-bound
// (reads 2 d bytes, writes d + 4).
#pragma once
#include "device.cuh"

namespace qsa {

template <int D>
__global__ void __launch_bounds__(256) quantize_kv_fp8_kernel(const __nv_bfloat16 *__restrict__ X,
                                                              uint8_t *__restrict__ codes,
                                                              float *__restrict__ scales, long rows)
{
    constexpr int V = D / 32;
    static_assert(V == 4, "rotated fp8 rows are 128 wide");
    const long row = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;   // whole warps
    const int lane = threadIdx.x & 31;
    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(X + row * D) + lane);
    float x[V];
    x[0] = __uint_as_float(raw.x << 16), x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    x[2] = __uint_as_float(raw.y << 16), x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    fwht_warp<V>(x);
    float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
    const float s = a > 0.f ? __fdiv_rn(a, 448.0f) : 0.f;
    uint32_t packed = 0;
    if (s > 0.f) {
        const uint16_t c01 = cvt_e4m3x2(__fdiv_rn(x[0], s), __fdiv_rn(x[1], s));
        const uint16_t c23 = cvt_e4m3x2(__fdiv_rn(x[2], s), __fdiv_rn(x[3], s));
        packed = (uint32_t)c01 | ((uint32_t)c23 << 16);
    }
    reinterpret_cast<uint32_t *>(codes + row * D)[lane] = packed;
    if (lane == 0) scales[row] = s;
}

}  // namespace qsa
