// libqsa.so -- host side of the C ABI declared in include/qsa.h.
// One translation unit holds every kernel (so the device status word is a
// single symbol) and the launch code: argument checks, TMA descriptor
// encoding, grid sizing and launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <climits>
#include <new>
#include <mutex>

#include "../../include/qsa.h"
#include "aggregate.cuh"
#include "compress.cuh"
#include "decode.cuh"
#include "device.cuh"
#include "prefill.cuh"
#include "quant.cuh"
#include "select.cuh"

namespace {

thread_local char g_last_error[512] = "";
std::atomic<unsigned long long> g_launches{0};

qsa_status fail(qsa_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

qsa_status check_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return QSA_OK;
}

// Called after each kernel launch of the library.
qsa_status launched(const char *what)
{
    qsa_status s = check_launch(what);
    if (s == QSA_OK) g_launches.fetch_add(1, std::memory_order_relaxed);
    return s;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDevicesSm = 128;

// ---------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D bf16 view [rows][cols] (cols contiguous) with 64 x 64 boxes, 128-byte swizzle.
qsa_status make_map_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows = 64)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled(2d) failed: %d", (int)r);
    return QSA_OK;
}

// 2-D byte view [rows][cols] (fp8 codes) with 64-row x 128-byte boxes, 128-byte swizzle.
qsa_status make_map_2d_u8(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled(2d, u8) failed: %d", (int)r);
    return QSA_OK;
}

// 3-D bf16 view of Q: [tokens][heads][d] with boxes (64 cols, G heads, TOK tokens).
qsa_status make_map_q(CUtensorMap *m, const void *base, uint64_t tokens, uint64_t heads, uint64_t d,
                      uint32_t box_heads, uint32_t box_tokens)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {d, heads, tokens};
    cuuint64_t strides[2] = {d * 2, heads * d * 2};
    cuuint32_t box[3] = {64, box_heads, box_tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled(3d) failed: %d", (int)r);
    return QSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool supported_d(int d) { return d == 64 || d == 128; }

// ------------------------------------------------------- select geometry
struct SelectPlan {
    int NR, CH, maxchunks;
    bool wide;            // prefill rows each selected whole by one 1024-thread CTA
    int TS;               // prefill rows: score-table row stride (floats)
    size_t qbar_bytes, part_bytes, table_bytes;
};

int sm_count();
constexpr int kWideMax = 24576;   // candidates of one row whose keys (192 KiB) fit one CTA

SelectPlan plan_select(int B, int Hkv, int Tq, int q_pos0, int qblk, int d)
{
    SelectPlan p;
    p.NR = (Tq + qblk - 1) / qblk;
    const int Dmax = (q_pos0 + Tq - 1) / 64;
    const int ncand = Dmax > 1 ? Dmax - 1 : 0;
    const long rows = (long)B * Hkv * p.NR;
    int CH = 2048;
    // enough CTAs to cover the SMs a few times over
    while (CH > 512 && rows * ((ncand + CH - 1) / CH) < 4 * 148) CH /= 2;
    // prefill rows longer than one chunk, few enough for about one wave of
    // 1024-thread CTAs, are selected whole from the score table by one CTA
    // each (the keys in shared memory), with no chunk lists and no merge
    p.wide = qblk == 64 && ncand > CH && ncand <= kWideMax && rows <= 2L * sm_count();
    if (p.wide) CH = (ncand + 3) / 4 * 4;
    p.CH = CH;
    p.maxchunks = ncand > 0 ? (ncand + CH - 1) / CH : 1;
    p.qbar_bytes = align256((size_t)rows * d * sizeof(float));
    p.part_bytes = p.maxchunks > 1 ? align256((size_t)rows * p.maxchunks * qsa::kMaxChosen * 8) : 0;
    // prefill rows (qblk = 64) are scored 8 rows at a time into a table
    // whose rows hold candidates 1 .. Dmax - 1 at their block index
    p.TS = qblk == 64 ? (Dmax + 3) / 4 * 4 : 0;
    p.table_bytes = qblk == 64 ? align256((size_t)rows * p.TS * sizeof(float)) : 0;
    return p;
}

// Per-token rows (qblk = 1) take the one-launch path when every row's
// candidates fit in 8 chunks of at most 8192: the chunks of a row form a
// cluster of NCH CTAs (enough CTAs to cover the SMs about 4 times).
struct TokenPlan {
    bool use;
    int NCH, CH;
};

int sm_count();

TokenPlan plan_token(int B, int Hkv, int Tq, int q_pos0, int qblk)
{
    TokenPlan p = {false, 1, 32};
    if (qblk != 1 || Tq > 65535 || (long)B * Hkv > 65535) return p;
    const int Dmax = (q_pos0 + Tq - 1) / 64;
    const int ncand = Dmax > 1 ? Dmax - 1 : 0;
    if (ncand > 8 * 8192) return p;
    const long rows = (long)B * Hkv * Tq;
    long nch = (4L * sm_count() + rows - 1) / rows;
    nch = nch > 8 ? 8 : nch;
    const long by_size = (ncand + 31) / 32;          // at least 32 candidates per chunk
    nch = nch > by_size ? by_size : nch;
    const long need = (ncand + 8191) / 8192;         // at most 8192 per chunk
    nch = nch < need ? need : nch;
    nch = nch < 1 ? 1 : nch;
    p.use = true;
    p.NCH = (int)nch;
    const int per = (ncand + p.NCH - 1) / p.NCH;
    p.CH = per < 32 ? 32 : (per + 31) / 32 * 32;
    return p;
}

// ------------------------------------------------------- decode geometry
int sm_count()
{
    static int cache[kMaxDevicesSm] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevicesSm) return 148;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// CTAs per (sequence, group) row: about CTAS_PER_SM * SMs CTAs over all
// rows without a second wave; at most 8 (one portable cluster) and at
// least one selected slot per CTA.
struct DecodePlan {
    int P, spc;
};

DecodePlan plan_decode(int rows, int topk, int nsm, int ctas_per_sm, int max_p = 8)
{
    int P = (ctas_per_sm * nsm) / rows;
    P = P < 1 ? 1 : P;
    P = P > max_p ? max_p : P;
    P = P > topk ? topk : P;
    DecodePlan p;
    p.spc = (topk + P - 1) / P;
    p.P = (topk + p.spc - 1) / p.spc;
    return p;
}

template <typename K>
qsa_status set_smem(K kernel, int bytes)
{
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return check_launch("cudaFuncSetAttribute");
    return QSA_OK;
}

// ------------------------------------------------------------ launchers
// Ragged / paged caches: per-sequence lengths (decode, compress) or first
// query positions (prefill) and the block table (device arrays; null for the
// contiguous, one-length layout).
struct Paging {
    const int32_t *seq_lens = nullptr;
    const int32_t *q_pos = nullptr;
    const int32_t *block_table = nullptr;
    int max_blocks = 0, num_pages = 0;
};

// A rank's share of a sharded cache: the blocks [lo, hi) it holds (block j
// at row 64 (j - lo) of its cache); partial: rows with none of their blocks
// here are not an error (O = 0, lse = -inf).  The default is the whole cache.
struct Ownership {
    int lo = 0, hi = INT_MAX, partial = 0;
};

template <int D, int G>
qsa_status launch_prefill(const void *Q, const void *K, const void *V, const int32_t *idx, void *O,
                          float *lse, int B, int Hq, int Hkv, int Tq, int q_pos0, int T_kv_max,
                          int topk, float sm_scale, cudaStream_t s, const Paging &pg = Paging(),
                          const Ownership &own = Ownership())
{
    using C = qsa::PrefillCfg<D, G>;
    CUtensorMap mq, mk, mv;
    qsa_status st;
    if ((st = make_map_q(&mq, Q, (uint64_t)B * Tq, Hq, D, G, C::TOK)) != QSA_OK) return st;
    // cache rows: [B][Hkv][T_kv_max], or [num_pages][Hkv][64] when paged
    const uint64_t nrows = pg.block_table ? (uint64_t)pg.num_pages * Hkv * 64 : (uint64_t)B * Hkv * T_kv_max;
    if ((st = make_map_2d(&mk, K, nrows, D)) != QSA_OK) return st;
    if ((st = make_map_2d(&mv, V, nrows, D)) != QSA_OK) return st;
    auto kern = qsa::sparse_attn_prefill_kernel<D, G>;
    // the kernel's setmaxnreg split waits without a limit unless every
    // thread starts with C::REG_LAUNCH registers: refuse any other build
    {
        static int regs = 0;
        if (!regs) {
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return check_launch("cudaFuncGetAttributes");
            regs = fa.numRegs;
        }
        if (regs != C::REG_LAUNCH)
            return fail(QSA_ERR_UNSUPPORTED, "sparse_attn_prefill_kernel built with %d registers per thread, "
                        "its register split needs %d", regs, C::REG_LAUNCH);
    }
    if ((st = set_smem(kern, C::SMEM_REQUEST)) != QSA_OK) return st;
    // persistent: one CTA per SM (never more than there are work units)
    const long units = (long)((Tq + 63) / 64) * C::TILES * B * Hkv;
    const int grid = (int)std::min<long>(units, sm_count());
    kern<<<grid, C::THREADS, C::SMEM_REQUEST, s>>>(mq, mk, mv, idx, (__nv_bfloat16 *)O, lse, Tq, Hq, Hkv,
                                                   B * Hkv, q_pos0, T_kv_max, topk,
                                                   sm_scale * 1.4426950408889634f, pg.q_pos, pg.block_table,
                                                   pg.max_blocks, pg.num_pages, own.lo, own.hi, own.partial);
    return launched("sparse_attn_prefill_kernel");
}

template <int D, int G, bool FP8 = false>
qsa_status launch_decode(const void *q, const void *K, const void *V, const int32_t *idx, void *o,
                         int B, int Hq, int Hkv, int L, int T_kv_max, int topk, float sm_scale,
                         cudaStream_t s, const Paging &pg = Paging(), const float *k_scales = nullptr,
                         const float *v_scales = nullptr)
{
    using C = qsa::DecodeCfg<D, FP8>;
    CUtensorMap mk, mv;
    qsa_status st;
    // cache rows: [B][Hkv][T_kv_max], or [num_pages][Hkv][64] when paged
    const uint64_t nrows = pg.block_table ? (uint64_t)pg.num_pages * Hkv * 64 : (uint64_t)B * Hkv * T_kv_max;
    if constexpr (FP8) {
        if ((st = make_map_2d_u8(&mk, K, nrows, D)) != QSA_OK) return st;
        if ((st = make_map_2d_u8(&mv, V, nrows, D)) != QSA_OK) return st;
    } else {
        if ((st = make_map_2d(&mk, K, nrows, D)) != QSA_OK) return st;
        if ((st = make_map_2d(&mv, V, nrows, D)) != QSA_OK) return st;
    }
    auto kern = qsa::decode_kernel<D, G, FP8>;
    DecodePlan p = plan_decode(B * Hkv, topk, sm_count(), C::CTAS_PER_SM);
    // the ring, then the merge inbox for this cluster size; a cluster size
    // whose inbox would leave no room for C::CTAS_PER_SM CTAs per SM gives
    // way to the next smaller one
    {
        cudaFuncAttributes fa;
        int dev = 0, per_sm = 0, reserved = 0;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
            return check_launch("decode_kernel attributes");
        auto fits = [&](int P) {
            return (long)C::CTAS_PER_SM * ((long)fa.sharedSizeBytes + C::SMEM_BYTES + C::inbox_bytes(G, P) + reserved) <=
                   per_sm;
        };
        while (p.P > 1 && !fits(p.P)) p = plan_decode(B * Hkv, topk, sm_count(), C::CTAS_PER_SM, p.P - 1);
    }
    const int smem = C::SMEM_BYTES + C::inbox_bytes(G, p.P);
    if ((st = set_smem(kern, smem)) != QSA_OK) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.P, B * Hkv, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait()
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mk, mv, (const __nv_bfloat16 *)q, idx, (__nv_bfloat16 *)o, Hq,
                                       Hkv, L, T_kv_max, topk, p.spc, sm_scale * 1.4426950408889634f,
                                       pg.seq_lens, pg.block_table, pg.max_blocks, pg.num_pages, k_scales,
                                       v_scales);
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "decode_kernel launch: %s", cudaGetErrorString(e));
    return launched("decode_kernel");
}

template <int D, typename KcT, bool SOFTMAX = false>
qsa_status launch_select_token_d(const void *Q, const KcT *Kc, int32_t *idx, int B, int Hq, int Hkv, int Tq,
                                 int q_pos0, int nblk_max, int topk, float sm_scale, const TokenPlan &tp,
                                 cudaStream_t s, const int32_t *seq_lens)
{
    auto kern = [] {
        if constexpr (SOFTMAX) return qsa::select_token_softmax_kernel<D, KcT>;
        else return qsa::select_token_kernel<D, KcT>;
    }();
    // keys; the softmax-sum path also keeps its chunk's logits (8 x (CH + 1) floats) when CH is short enough
    const int smem = tp.CH * 8 + (SOFTMAX && tp.CH <= qsa::kSoftmaxZCap ? 8 * (tp.CH + 1) * 4 : 0);
    qsa_status st;
    if ((st = set_smem(kern, smem)) != QSA_OK) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tp.NCH, Tq, B * Hkv);
    cfg.blockDim = dim3(qsa::kSelThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = tp.NCH;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see grid_dependency_wait()
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, (const __nv_bfloat16 *)Q, Kc, idx, nblk_max, Tq, Hq, Hkv,
                                       q_pos0, topk, sm_scale, tp.CH, seq_lens);
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "select_token_kernel launch: %s", cudaGetErrorString(e));
    return launched(SOFTMAX ? "select_token_softmax_kernel" : "select_token_kernel");
}

template <typename KcT, bool SOFTMAX = false>
qsa_status launch_select_token(const void *Q, const KcT *Kc, int32_t *idx, int B, int Hq, int Hkv, int Tq,
                               int q_pos0, int nblk_max, int d, int topk, float sm_scale, const TokenPlan &tp,
                               cudaStream_t s, const int32_t *seq_lens = nullptr)
{
    if (d == 128)
        return launch_select_token_d<128, KcT, SOFTMAX>(Q, Kc, idx, B, Hq, Hkv, Tq, q_pos0, nblk_max, topk, sm_scale,
                                                        tp, s, seq_lens);
    return launch_select_token_d<64, KcT, SOFTMAX>(Q, Kc, idx, B, Hq, Hkv, Tq, q_pos0, nblk_max, topk, sm_scale, tp,
                                                   s, seq_lens);
}

template <bool WEIGHT>
__global__ void selftest_exp2_kernel(const float *__restrict__ x, float *__restrict__ y, int n)
{
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    auto e2 = [](float a, float b) {
        return WEIGHT ? qsa::exp2_poly5_x2(qsa::f2_pack(a, b)) : qsa::exp2_poly_x2(qsa::f2_pack(a, b));
    };
    if (i + 1 < n) {
        float a, b;
        qsa::f2_unpack(e2(x[i], x[i + 1]), a, b);
        y[i] = a;
        y[i + 1] = b;
    } else if (i < n) {
        float a, b;
        qsa::f2_unpack(e2(x[i], 0.f), a, b);
        y[i] = a;
    }
}

__global__ void selftest_wait_kernel(uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        qsa::mbar_init(&bar, 1);   // nothing ever arrives
        qsa::fence_barrier_init();
    }
    __syncthreads();
    qsa::mbar_wait(&bar, 0, &abort_flag, 99, limit_ns);
}

}  // namespace

// ------------------------------------------- allocation-free selection
// Scratch of qsa_score_select_noalloc: a file-scope device array that every
// GPU loading the library holds until the process exits.  Host code only
// sees a host-side stand-in for it, so the device address is looked up once
// per device (with that device current) and cached.
static __device__ __align__(256) uint8_t g_select_scratch[QSA_SELECT_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 128;

qsa_status select_scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return check_launch("cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(QSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess || !p)
            return fail(QSA_ERR_CUDA, "cudaGetSymbolAddress(select scratch): %s", cudaGetErrorString(e));
        addr[dev] = p;
    }
    *out = addr[dev];
    return QSA_OK;
}

}  // namespace

namespace {

template <typename KcT>
qsa_status compress_keys_impl(const char *name, const void *K, KcT *Kc, int B, int Hkv, int T_kv_max, int d,
                              int blk_begin, int blk_end, qsa_stream_t stream, const Paging &pg = Paging())
{
    if (!K || !Kc) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hkv <= 0 || T_kv_max <= 0 || T_kv_max % 64)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    const int nblk_max = T_kv_max / 64;
    if (blk_begin < 0 || blk_end < blk_begin || blk_end > nblk_max)
        return fail(QSA_ERR_INVALID_ARG, "%s: block range [%d,%d) outside [0,%d]", name, blk_begin,
                    blk_end, nblk_max);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (!aligned16(K) || !aligned16(Kc)) return fail(QSA_ERR_INVALID_ARG, "%s: misaligned", name);
    const int nblk = blk_end - blk_begin;
    if (nblk == 0) return QSA_OK;
    const long grid = (long)B * Hkv * nblk;
    if (grid >= (1L << 31)) return fail(QSA_ERR_UNSUPPORTED, "%s: too many blocks", name);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 128)
        qsa::compress_keys_kernel<128, KcT><<<(unsigned)grid, 128, 0, s>>>((const __nv_bfloat16 *)K, Kc, T_kv_max,
                                                                      nblk_max, blk_begin, nblk, pg.block_table,
                                                                      pg.seq_lens, Hkv, pg.num_pages);
    else
        qsa::compress_keys_kernel<64, KcT><<<(unsigned)grid, 128, 0, s>>>((const __nv_bfloat16 *)K, Kc, T_kv_max,
                                                                     nblk_max, blk_begin, nblk, pg.block_table,
                                                                     pg.seq_lens, Hkv, pg.num_pages);
    return launched("compress_keys_kernel");
}


// Score-table launch: one CTA per (64-row tile, 64-candidate tile) of the
// candidates in [lo, hi) up to the last row's diagonal.
struct TableLaunch {
    dim3 grid;
    int smem;
};

TableLaunch plan_table(int B, int Hkv, int Tq, int q_pos0, int lo, int hi, int d)
{
    constexpr int T = qsa::kTableTile;
    const int NR = (Tq + 63) / 64;
    const int Dmax = (q_pos0 + Tq - 1) / 64;
    const int n = std::min(Dmax, hi) - lo;
    TableLaunch tl;
    tl.grid = dim3((unsigned)std::max(1, (n + T - 1) / T), (unsigned)((NR + T - 1) / T), (unsigned)(B * Hkv));
    tl.smem = 2 * T * (d + 4) * (int)sizeof(float);
    return tl;
}

// Pooling launch: the 16-byte column chunks of a token's heads, times up to
// four token splits for rows of several tokens (at most 1024 threads).
struct PoolLaunch {
    int threads, TS, smem;
};

PoolLaunch plan_pool(int Hq, int d, int qblk, long ctas)
{
    const int nc = ((Hq * d / 8) + 31) / 32 * 32;
    // split tokens only when the rows' CTAs are too few to fill the GPU
    int TS = (qblk > 1 && ctas < 2L * sm_count()) ? 1024 / nc : 1;
    TS = TS > 4 ? 4 : (TS < 1 ? 1 : TS);
    return {nc * TS, TS, TS * Hq * d * (int)sizeof(float)};
}

// Pooling, then scoring and selection: prefill rows through the score
// table (score_table_kernel, then score_select_kernel from the table),
// long per-token rows by score_select_kernel's own scoring.
template <int D, typename KcT>
qsa_status launch_score_select(const void *Q, const KcT *Kc, int32_t *idx, float *Qbar, uint64_t *part, float *table,
                               const SelectPlan &p, dim3 pgrid, const PoolLaunch &pl, dim3 sgrid, int ssmem,
                               int B, int Hq, int Hkv, int Tq, int q_pos0, int qblk, int nblk_max, int topk,
                               float sm_scale, const int32_t *q_pos, cudaStream_t s)
{
    qsa_status st;
    if ((st = set_smem(qsa::pool_queries_kernel<D>, pl.smem)) != QSA_OK) return st;
    qsa::pool_queries_kernel<D><<<pgrid, pl.threads, pl.smem, s>>>((const __nv_bfloat16 *)Q, Qbar, Tq, Hq, Hkv, qblk,
                                                                   pl.TS);
    if ((st = launched("pool_queries_kernel")) != QSA_OK) return st;
    if (qblk == 64) {
        const TableLaunch tl = plan_table(B, Hkv, Tq, q_pos0, 1, INT_MAX, D);
        if ((st = set_smem(qsa::score_table_kernel<D, KcT>, tl.smem)) != QSA_OK) return st;
        qsa::score_table_kernel<D, KcT><<<tl.grid, 256, tl.smem, s>>>(Qbar, Kc, table, nblk_max, Tq, q_pos0, p.TS,
                                                                      sm_scale, Hkv, q_pos, 1, INT_MAX, 0, nblk_max, 0);
        if ((st = launched("score_table_kernel")) != QSA_OK) return st;
        if (p.wide) {
            auto kern = qsa::score_select_kernel<D, KcT, true, 1024>;
            if ((st = set_smem(kern, ssmem)) != QSA_OK) return st;
            kern<<<sgrid, 1024, ssmem, s>>>(nullptr, Kc, idx, part, nblk_max, Tq, q_pos0, qblk, topk, sm_scale, p.CH,
                                            p.maxchunks, Hkv, q_pos, table, p.TS);
        } else {
            auto kern = qsa::score_select_kernel<D, KcT, true>;
            if ((st = set_smem(kern, ssmem)) != QSA_OK) return st;
            kern<<<sgrid, qsa::kSelThreads, ssmem, s>>>(nullptr, Kc, idx, part, nblk_max, Tq, q_pos0, qblk, topk,
                                                        sm_scale, p.CH, p.maxchunks, Hkv, q_pos, table, p.TS);
        }
    } else {
        auto kern = qsa::score_select_kernel<D, KcT>;
        if ((st = set_smem(kern, ssmem)) != QSA_OK) return st;
        kern<<<sgrid, qsa::kSelThreads, ssmem, s>>>(Qbar, Kc, idx, part, nblk_max, Tq, q_pos0, qblk, topk, sm_scale,
                                                    p.CH, p.maxchunks, Hkv, q_pos, nullptr, 0);
    }
    return launched("score_select_kernel");
}

template <typename KcT>
qsa_status score_select_impl(const char *name, const void *Q, const KcT *Kc, int32_t *idx, int B, int Hq, int Hkv,
                             int Tq, int q_pos0, int qblk, int T_kv_max, int d, int topk, float sm_scale,
                             void *workspace, size_t workspace_bytes, qsa_stream_t stream,
                             const int32_t *q_pos = nullptr)
{
    if (!Q || !Kc || !idx) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || T_kv_max <= 0 || T_kv_max % 64 ||
        Hq % Hkv)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if (qblk != 1 && qblk != 64) return fail(QSA_ERR_UNSUPPORTED, "%s: qblk=%d", name, qblk);
    if (qblk == 64 && q_pos0 % 64)
        return fail(QSA_ERR_INVALID_ARG, "%s: q_pos0 must be a multiple of 64 when qblk=64", name);
    if ((long)q_pos0 + Tq > T_kv_max) return fail(QSA_ERR_INVALID_ARG, "%s: queries past the cache", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    if ((long)Hq * d / 8 > 1024) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq*d too large", name);
    if (!aligned16(Q) || !aligned16(Kc) || !aligned16(idx))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const TokenPlan tp = plan_token(B, Hkv, Tq, q_pos0, qblk);
    if (tp.use) return launch_select_token(Q, Kc, idx, B, Hq, Hkv, Tq, q_pos0, T_kv_max / 64, d, topk, sm_scale,
                                           tp, s);
    const SelectPlan p = plan_select(B, Hkv, Tq, q_pos0, qblk, d);
    if (p.maxchunks * qsa::kMaxChosen * 8 > 200 * 1024)
        return fail(QSA_ERR_UNSUPPORTED, "%s: context too long", name);
    const size_t need = p.qbar_bytes + p.part_bytes + p.table_bytes;
    if (!workspace || workspace_bytes < need || !aligned16(workspace))
        return fail(QSA_ERR_WORKSPACE, "%s: workspace needs %zu bytes", name, need);
    float *Qbar = static_cast<float *>(workspace);
    uint64_t *part = reinterpret_cast<uint64_t *>(static_cast<uint8_t *>(workspace) + p.qbar_bytes);
    float *table = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + p.qbar_bytes + p.part_bytes);
    const int nblk_max = T_kv_max / 64;
    const PoolLaunch pl = plan_pool(Hq, d, qblk, (long)p.NR * B);
    dim3 pgrid(p.NR, B), sgrid(p.maxchunks, p.NR, B * Hkv), mgrid(p.NR, B * Hkv);
    const int ssmem = p.CH * 8;
    qsa_status st;
    if (d == 128) st = launch_score_select<128, KcT>(Q, Kc, idx, Qbar, part, table, p, pgrid, pl,
                                                      sgrid, ssmem, B, Hq, Hkv, Tq, q_pos0, qblk,
                                                      nblk_max, topk, sm_scale, q_pos, s);
    else st = launch_score_select<64, KcT>(Q, Kc, idx, Qbar, part, table, p, pgrid, pl,
                                           sgrid, ssmem, B, Hq, Hkv, Tq, q_pos0, qblk, nblk_max, topk, sm_scale,
                                           q_pos, s);
    if (st != QSA_OK) return st;
    if (p.maxchunks > 1) {
        const int msmem = p.maxchunks * qsa::kMaxChosen * 8;
        if ((st = set_smem(qsa::merge_select_kernel, msmem)) != QSA_OK) return st;
        qsa::merge_select_kernel<<<mgrid, qsa::kSelThreads, msmem, s>>>(part, idx, Tq, q_pos0, qblk, topk, p.CH,
                                                                       p.maxchunks, Hkv, nblk_max, q_pos);
        if ((st = launched("merge_select_kernel")) != QSA_OK) return st;
    }
    return QSA_OK;
}


template <int G>
qsa_status launch_prefill_agg(const void *Q, const void *Kc, float *scores, float *stats, int B, int Hq, int Hkv,
                              int Tq, int q_pos0, int nblk, int NR, float sm_scale, int aggregator, cudaStream_t s)
{
    qsa_status st;
    CUtensorMap mq, mk;
    if ((st = make_map_2d(&mk, Kc, (uint64_t)B * Hkv * nblk, 128, 128)) != QSA_OK) return st;
    if (aggregator == QSA_AGG_SOFTMAX_SUM) {
        using S = qsa::SoftmaxStatsCfg<G>;
        CUtensorMap mq1, mk1;
        if ((st = make_map_q(&mq1, Q, (uint64_t)B * Tq, Hq, 128, G, S::TOKM)) != QSA_OK) return st;
        if ((st = make_map_2d(&mk1, Kc, (uint64_t)B * Hkv * nblk, 128, 256)) != QSA_OK) return st;
        if ((st = set_smem(qsa::block_softmax_stats_kernel<G>, S::SMEM_BYTES)) != QSA_OK) return st;
        // persistent: one CTA per SM over the (sequence and group, query block, M tile) units
        const long nunits = (long)NR * S::NMT * B * Hkv;
        if (nunits >= (1L << 31)) return fail(QSA_ERR_UNSUPPORTED, "softmax statistics: too many rows");
        const int grid = (int)std::min<long>(nunits, sm_count());
        qsa::block_softmax_stats_kernel<G><<<grid, S::THREADS, S::SMEM_BYTES, s>>>(
            mq1, mk1, stats, Tq, q_pos0, nblk, Hkv, sm_scale, NR, (int)nunits);
        if ((st = launched("block_softmax_stats_kernel")) != QSA_OK) return st;
    }
    using C = qsa::TokenScoresCfg<G>;
    if ((st = make_map_q(&mq, Q, (uint64_t)B * Tq, Hq, 128, G, C::TOKN)) != QSA_OK) return st;
    // persistent: one CTA per SM over the (sequence and group, query block) units
    const long nunits = (long)NR * B * Hkv;
    const int grid = (int)std::min<long>(nunits, sm_count());
    if (aggregator == QSA_AGG_SOFTMAX_SUM) {
        if ((st = set_smem(qsa::block_softmax_scores_kernel<G>, C::SMEM_BYTES)) != QSA_OK) return st;
        qsa::block_softmax_scores_kernel<G><<<grid, C::THREADS, C::SMEM_BYTES, s>>>(
            mq, mk, scores, stats, Tq, q_pos0, nblk, Hkv, sm_scale, NR, (int)nunits);
        return launched("block_softmax_scores_kernel");
    }
    if ((st = set_smem(qsa::block_max_scores_kernel<G>, C::SMEM_BYTES)) != QSA_OK) return st;
    qsa::block_max_scores_kernel<G><<<grid, C::THREADS, C::SMEM_BYTES, s>>>(mq, mk, scores, Tq, q_pos0, nblk, Hkv,
                                                                           sm_scale, NR, (int)nunits);
    return launched("block_max_scores_kernel");
}
}  // namespace

// ------------------------------------------- host-buffer prefill pipeline
// Two device buffer sets and three streams; step k uses set k % 2.
struct qsa_prefill_pipeline {
    struct Set {
        void *Q = nullptr, *K = nullptr, *V = nullptr, *O = nullptr, *ws = nullptr;
        float *Kc = nullptr;
        int32_t *idx = nullptr;
        cudaEvent_t up = nullptr, done = nullptr, down = nullptr;
        bool used = false;
    };
    int B = 0, Hq = 0, Hkv = 0, Tq = 0, q_pos0 = 0, T_kv_max = 0, d = 0, topk = 0;
    float sm_scale = 0.f;
    size_t q_bytes = 0, kv_bytes = 0, kc_bytes = 0, idx_bytes = 0, ws_bytes = 0;
    Set set[2];
    cudaStream_t s_in = nullptr, s_cmp = nullptr, s_out = nullptr;
    long k = 0;
};

namespace {
void pipeline_free(qsa_prefill_pipeline *p)
{
    if (!p) return;
    for (auto *s : {p->s_in, p->s_cmp, p->s_out})
        if (s) cudaStreamSynchronize(s);
    for (auto &x : p->set) {
        for (void *m : {x.Q, x.K, x.V, x.O, x.ws, (void *)x.Kc, (void *)x.idx})
            if (m) cudaFree(m);
        for (cudaEvent_t e : {x.up, x.done, x.down})
            if (e) cudaEventDestroy(e);
    }
    for (auto *s : {p->s_in, p->s_cmp, p->s_out})
        if (s) cudaStreamDestroy(s);
    delete p;
}
}  // namespace

// ===================================================================== C ABI
extern "C" {

qsa_status qsa_compress_keys(const void *K, float *Kc, int B, int Hkv, int T_kv_max, int d, int blk_begin,
                             int blk_end, qsa_stream_t stream)
{
    return compress_keys_impl("qsa_compress_keys", K, Kc, B, Hkv, T_kv_max, d, blk_begin, blk_end, stream);
}

qsa_status qsa_compress_keys_bf16(const void *K, void *Kc, int B, int Hkv, int T_kv_max, int d, int blk_begin,
                                  int blk_end, qsa_stream_t stream)
{
    return compress_keys_impl("qsa_compress_keys_bf16", K, static_cast<__nv_bfloat16 *>(Kc), B, Hkv, T_kv_max, d,
                              blk_begin, blk_end, stream);
}

qsa_status qsa_compress_keys_paged(const void *K_pages, const int32_t *block_table, const int32_t *seq_lens,
                                   float *Kc, int B, int Hkv, int max_blocks, int num_pages, int d, int blk_begin,
                                   int blk_end, qsa_stream_t stream)
{
    if (!block_table || !seq_lens) return fail(QSA_ERR_INVALID_ARG, "qsa_compress_keys_paged: null pointer");
    if (max_blocks <= 0 || num_pages <= 0 || Hkv <= 0 || (long)num_pages * Hkv * 64 >= (1L << 31) ||
        (long)max_blocks * 64 >= (1L << 31))
        return fail(QSA_ERR_UNSUPPORTED, "qsa_compress_keys_paged: bad page geometry");
    Paging pg;
    pg.seq_lens = seq_lens;
    pg.block_table = block_table;
    pg.max_blocks = max_blocks;
    pg.num_pages = num_pages;
    return compress_keys_impl("qsa_compress_keys_paged", K_pages, Kc, B, Hkv, 64 * max_blocks, d, blk_begin, blk_end,
                              stream, pg);
}

size_t qsa_score_select_workspace(int B, int Hq, int Hkv, int Tq, int q_pos0, int qblk, int d, int topk)
{
    (void)Hq;
    (void)topk;
    if (B <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || (qblk != 1 && qblk != 64) || !supported_d(d)) return 0;
    if (plan_token(B, Hkv, Tq, q_pos0, qblk).use) return 0;
    const SelectPlan p = plan_select(B, Hkv, Tq, q_pos0, qblk, d);
    return p.qbar_bytes + p.part_bytes + p.table_bytes;
}

qsa_status qsa_score_select(const void *Q, const float *Kc, int32_t *idx, int B, int Hq, int Hkv, int Tq,
                            int q_pos0, int qblk, int T_kv_max, int d, int topk, float sm_scale,
                            void *workspace, size_t workspace_bytes, qsa_stream_t stream)
{
    return score_select_impl("qsa_score_select", Q, Kc, idx, B, Hq, Hkv, Tq, q_pos0, qblk, T_kv_max, d, topk,
                             sm_scale, workspace, workspace_bytes, stream);
}

qsa_status qsa_score_select_bf16(const void *Q, const void *Kc, int32_t *idx, int B, int Hq, int Hkv, int Tq,
                                 int q_pos0, int qblk, int T_kv_max, int d, int topk, float sm_scale,
                                 void *workspace, size_t workspace_bytes, qsa_stream_t stream)
{
    return score_select_impl("qsa_score_select_bf16", Q, static_cast<const __nv_bfloat16 *>(Kc), idx, B, Hq, Hkv,
                             Tq, q_pos0, qblk, T_kv_max, d, topk, sm_scale, workspace, workspace_bytes, stream);
}

qsa_status qsa_score_select_ragged(const void *Q, const float *Kc, const int32_t *seq_lens, int32_t *idx, int B,
                                   int Hq, int Hkv, int max_blocks, int max_len, int d, int topk, float sm_scale,
                                   qsa_stream_t stream)
{
    const char *name = "qsa_score_select_ragged";
    if (!Q || !Kc || !seq_lens || !idx) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || max_blocks <= 0 || max_len < 1 ||
        (long)max_len > 64L * max_blocks)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    if ((long)Hq * d / 8 > 1024) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq*d too large", name);
    if (!aligned16(Q) || !aligned16(Kc) || !aligned16(idx) || (reinterpret_cast<uintptr_t>(seq_lens) & 3))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    const TokenPlan tp = plan_token(B, Hkv, 1, max_len - 1, 1);
    if (!tp.use) return fail(QSA_ERR_UNSUPPORTED, "%s: more candidates than one cluster of chunks holds", name);
    return launch_select_token(Q, Kc, idx, B, Hq, Hkv, 1, max_len - 1, max_blocks, d, topk, sm_scale, tp,
                               reinterpret_cast<cudaStream_t>(stream), seq_lens);
}

qsa_status qsa_score_select_token_agg(const void *Q, const float *Kc, const int32_t *seq_lens, int32_t *idx, int B,
                                      int Hq, int Hkv, int Tq, int q_pos0, int max_blocks, int d, int topk,
                                      float sm_scale, int aggregator, qsa_stream_t stream)
{
    const char *name = "qsa_score_select_token_agg";
    if (!Q || !Kc || !idx) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (aggregator != QSA_AGG_MEAN && aggregator != QSA_AGG_MAX && aggregator != QSA_AGG_SOFTMAX_SUM)
        return fail(QSA_ERR_INVALID_ARG, "%s: aggregator=%d", name, aggregator);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Tq <= 0 || q_pos0 < 0 || max_blocks <= 0 ||
        (long)q_pos0 + Tq > 64L * max_blocks || (seq_lens && Tq != 1))
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    if ((long)Hq * d / 8 > 1024 || Hq / Hkv > 8) return fail(QSA_ERR_UNSUPPORTED, "%s: group too large", name);
    if (!aligned16(Q) || !aligned16(Kc) || !aligned16(idx) || (reinterpret_cast<uintptr_t>(seq_lens) & 3))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    const TokenPlan tp = plan_token(B, Hkv, Tq, q_pos0, 1);
    if (!tp.use) return fail(QSA_ERR_UNSUPPORTED, "%s: more candidates than one cluster of chunks holds", name);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one token per row: its maximum over tokens is its mean
    if (aggregator == QSA_AGG_SOFTMAX_SUM)
        return launch_select_token<float, true>(Q, Kc, idx, B, Hq, Hkv, Tq, q_pos0, max_blocks, d, topk, sm_scale, tp,
                                                s, seq_lens);
    return launch_select_token<float>(Q, Kc, idx, B, Hq, Hkv, Tq, q_pos0, max_blocks, d, topk, sm_scale, tp, s,
                                      seq_lens);
}

size_t qsa_score_select_prefill_agg_workspace(int B, int Hq, int Hkv, int Tq, int q_pos0, int T_kv_max, int d,
                                              int topk, int aggregator)
{
    (void)topk;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || T_kv_max <= 0 || T_kv_max % 64 || d != 128)
        return 0;
    const SelectPlan p = plan_select(B, Hkv, Tq, q_pos0, 64, d);
    const size_t rows = (size_t)B * Hkv * p.NR;
    size_t bytes = align256(rows * (T_kv_max / 64) * sizeof(float)) + p.part_bytes;
    if (aggregator == QSA_AGG_SOFTMAX_SUM) bytes += align256(rows * 64 * (Hq / Hkv) * 2 * sizeof(float));
    return bytes;
}


qsa_status qsa_score_select_prefill_agg(const void *Q, const void *Kc, int32_t *idx, int B, int Hq, int Hkv, int Tq,
                                        int q_pos0, int T_kv_max, int d, int topk, float sm_scale, int aggregator,
                                        void *workspace, size_t workspace_bytes, qsa_stream_t stream)
{
    const char *name = "qsa_score_select_prefill_agg";
    if (!Q || !Kc || !idx) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (aggregator != QSA_AGG_MAX && aggregator != QSA_AGG_SOFTMAX_SUM)
        return fail(aggregator == QSA_AGG_MEAN ? QSA_ERR_UNSUPPORTED : QSA_ERR_INVALID_ARG,
                    "%s: aggregator=%d (the mean is qsa_score_select_bf16)", name, aggregator);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || T_kv_max <= 0 || T_kv_max % 64 || Hq % Hkv ||
        q_pos0 % 64 || (long)q_pos0 + Tq > T_kv_max)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if (d != 128) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d", name, G);
    const int nblk = T_kv_max / 64;
    if ((long)B * Hkv * nblk >= (1L << 31) || (long)B * Tq >= (1L << 31))
        return fail(QSA_ERR_UNSUPPORTED, "%s: too large", name);
    if (!aligned16(Q) || !aligned16(Kc) || !aligned16(idx) || (workspace && !aligned16(workspace)))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    const SelectPlan p = plan_select(B, Hkv, Tq, q_pos0, 64, d);
    if ((long)p.NR * 4 > 65535 || (long)B * Hkv > 65535) return fail(QSA_ERR_UNSUPPORTED, "%s: too many rows", name);
    if (p.maxchunks * qsa::kMaxChosen * 8 > 200 * 1024) return fail(QSA_ERR_UNSUPPORTED, "%s: context too long", name);
    const size_t rows = (size_t)B * Hkv * p.NR;
    const size_t score_bytes = align256(rows * nblk * sizeof(float));
    const size_t stat_bytes = aggregator == QSA_AGG_SOFTMAX_SUM ? align256(rows * 64 * G * 2 * sizeof(float)) : 0;
    if (!workspace || workspace_bytes < score_bytes + stat_bytes + p.part_bytes)
        return fail(QSA_ERR_WORKSPACE, "%s: workspace needs %zu bytes", name, score_bytes + stat_bytes + p.part_bytes);
    float *scores = static_cast<float *>(workspace);
    float *stats = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + score_bytes);
    uint64_t *part = reinterpret_cast<uint64_t *>(static_cast<uint8_t *>(workspace) + score_bytes + stat_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    qsa_status st = G == 8 ? launch_prefill_agg<8>(Q, Kc, scores, stats, B, Hq, Hkv, Tq, q_pos0, nblk, p.NR, sm_scale,
                                                   aggregator, s)
                           : launch_prefill_agg<4>(Q, Kc, scores, stats, B, Hq, Hkv, Tq, q_pos0, nblk, p.NR, sm_scale,
                                                   aggregator, s);
    if (st != QSA_OK) return st;
    const dim3 sgrid(p.maxchunks, p.NR, B * Hkv), mgrid(p.NR, B * Hkv);
    if (p.wide) {
        auto skern = qsa::score_select_kernel<128, __nv_bfloat16, true, 1024>;
        if ((st = set_smem(skern, p.CH * 8)) != QSA_OK) return st;
        skern<<<sgrid, 1024, p.CH * 8, s>>>(nullptr, static_cast<const __nv_bfloat16 *>(Kc), idx, part, nblk, Tq, q_pos0,
                                            64, topk, sm_scale, p.CH, p.maxchunks, Hkv, nullptr, scores, 0);
    } else {
        auto skern = qsa::score_select_kernel<128, __nv_bfloat16, true>;
        if ((st = set_smem(skern, p.CH * 8)) != QSA_OK) return st;
        skern<<<sgrid, qsa::kSelThreads, p.CH * 8, s>>>(nullptr, static_cast<const __nv_bfloat16 *>(Kc), idx, part,
                                                        nblk, Tq, q_pos0, 64, topk, sm_scale, p.CH, p.maxchunks, Hkv,
                                                        nullptr, scores, 0);
    }
    if ((st = launched("score_select_kernel")) != QSA_OK) return st;
    if (p.maxchunks > 1) {
        const int msmem = p.maxchunks * qsa::kMaxChosen * 8;
        if ((st = set_smem(qsa::merge_select_kernel, msmem)) != QSA_OK) return st;
        qsa::merge_select_kernel<<<mgrid, qsa::kSelThreads, msmem, s>>>(part, idx, Tq, q_pos0, 64, topk, p.CH,
                                                                       p.maxchunks, Hkv, nblk, nullptr);
        if ((st = launched("merge_select_kernel")) != QSA_OK) return st;
    }
    return QSA_OK;
}

qsa_status qsa_score_select_ragged_prefill(const void *Q, const float *Kc, const int32_t *q_pos, int32_t *idx,
                                           int B, int Hq, int Hkv, int Tq, int max_blocks, int max_pos, int d,
                                           int topk, float sm_scale, void *workspace, size_t workspace_bytes,
                                           qsa_stream_t stream)
{
    if (!q_pos) return fail(QSA_ERR_INVALID_ARG, "qsa_score_select_ragged_prefill: null pointer");
    if (max_pos < 0 || max_pos % 64 || max_blocks <= 0 || (long)max_blocks * 64 >= (1L << 31))
        return fail(QSA_ERR_INVALID_ARG, "qsa_score_select_ragged_prefill: bad max_pos / max_blocks");
    // planned for the furthest position; each row takes its own from q_pos
    return score_select_impl("qsa_score_select_ragged_prefill", Q, Kc, idx, B, Hq, Hkv, Tq, max_pos, 64,
                             64 * max_blocks, d, topk, sm_scale, workspace, workspace_bytes, stream, q_pos);
}

qsa_status qsa_score_select_noalloc(const void *Q, const float *Kc, int32_t *idx, int B, int Hq, int Hkv, int Tq,
                                    int q_pos0, int qblk, int T_kv_max, int d, int topk, float sm_scale,
                                    qsa_stream_t stream)
{
    const size_t need = qsa_score_select_workspace(B, Hq, Hkv, Tq, q_pos0, qblk, d, topk);
    if (need > QSA_SELECT_SCRATCH_BYTES)
        return fail(QSA_ERR_WORKSPACE,
                    "qsa_score_select_noalloc: this shape needs %zu bytes of scratch, the static buffer holds %zu; "
                    "use qsa_score_select with a caller workspace",
                    need, (size_t)QSA_SELECT_SCRATCH_BYTES);
    void *scratch = nullptr;
    qsa_status st = select_scratch_address(&scratch);
    if (st != QSA_OK) return st;
    return qsa_score_select(Q, Kc, idx, B, Hq, Hkv, Tq, q_pos0, qblk, T_kv_max, d, topk, sm_scale, scratch,
                            QSA_SELECT_SCRATCH_BYTES, stream);
}

qsa_status qsa_sparse_attn_prefill(const void *Q, const void *K, const void *V, const int32_t *idx, void *O,
                                   float *lse, int B, int Hq, int Hkv, int Tq, int q_pos0, int T_kv_max, int d,
                                   int topk, float sm_scale, qsa_stream_t stream)
{
    if (!Q || !K || !V || !idx || !O) return fail(QSA_ERR_INVALID_ARG, "qsa_sparse_attn_prefill: null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || T_kv_max <= 0 || T_kv_max % 64 || Hq % Hkv)
        return fail(QSA_ERR_INVALID_ARG, "qsa_sparse_attn_prefill: bad shape");
    if (q_pos0 % 64) return fail(QSA_ERR_INVALID_ARG, "qsa_sparse_attn_prefill: q_pos0 must be a multiple of 64");
    if ((long)q_pos0 + Tq > T_kv_max)
        return fail(QSA_ERR_INVALID_ARG, "qsa_sparse_attn_prefill: queries past the cache");
    if ((long)B * Hkv * T_kv_max >= (1L << 31) || (long)B * Tq >= (1L << 31))
        return fail(QSA_ERR_UNSUPPORTED, "qsa_sparse_attn_prefill: tensor too large");
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "qsa_sparse_attn_prefill: d=%d", d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "qsa_sparse_attn_prefill: topk=%d", topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "qsa_sparse_attn_prefill: Hq/Hkv=%d", G);
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(O))
        return fail(QSA_ERR_INVALID_ARG, "qsa_sparse_attn_prefill: misaligned pointer");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 128 && G == 8) return launch_prefill<128, 8>(Q, K, V, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_kv_max, topk, sm_scale, s);
    if (d == 128 && G == 4) return launch_prefill<128, 4>(Q, K, V, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_kv_max, topk, sm_scale, s);
    if (d == 64 && G == 8) return launch_prefill<64, 8>(Q, K, V, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_kv_max, topk, sm_scale, s);
    return launch_prefill<64, 4>(Q, K, V, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_kv_max, topk, sm_scale, s);
}

size_t qsa_decode_workspace(int B, int Hq, int Hkv, int d, int topk)
{
    (void)B;
    (void)Hq;
    (void)Hkv;
    (void)d;
    (void)topk;
    return 0;   // the split-K merge runs through distributed shared memory
}

qsa_status qsa_decode(const void *q, const void *K_cache, const void *V_cache, const int32_t *idx, void *o, int B,
                      int Hq, int Hkv, int L, int T_kv_max, int d, int topk, float sm_scale, void *workspace,
                      size_t workspace_bytes, qsa_stream_t stream)
{
    if (!q || !K_cache || !V_cache || !idx || !o) return fail(QSA_ERR_INVALID_ARG, "qsa_decode: null pointer");
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || T_kv_max <= 0 || T_kv_max % 64 || L > T_kv_max || Hq % Hkv)
        return fail(QSA_ERR_INVALID_ARG, "qsa_decode: bad shape");
    if ((long)B * Hkv * T_kv_max >= (1L << 31)) return fail(QSA_ERR_UNSUPPORTED, "qsa_decode: cache too large");
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "qsa_decode: d=%d", d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "qsa_decode: topk=%d", topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "qsa_decode: Hq/Hkv=%d", G);
    if (!aligned16(q) || !aligned16(K_cache) || !aligned16(V_cache) || !aligned16(idx) || !aligned16(o))
        return fail(QSA_ERR_INVALID_ARG, "qsa_decode: misaligned pointer");
    (void)workspace;
    (void)workspace_bytes;
    if (B * Hkv > 65535) return fail(QSA_ERR_UNSUPPORTED, "qsa_decode: more than 65535 (sequence, group) rows");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 128 && G == 8) return launch_decode<128, 8>(q, K_cache, V_cache, idx, o, B, Hq, Hkv, L, T_kv_max, topk, sm_scale, s);
    if (d == 128 && G == 4) return launch_decode<128, 4>(q, K_cache, V_cache, idx, o, B, Hq, Hkv, L, T_kv_max, topk, sm_scale, s);
    if (d == 64 && G == 8) return launch_decode<64, 8>(q, K_cache, V_cache, idx, o, B, Hq, Hkv, L, T_kv_max, topk, sm_scale, s);
    return launch_decode<64, 4>(q, K_cache, V_cache, idx, o, B, Hq, Hkv, L, T_kv_max, topk, sm_scale, s);
}

qsa_status qsa_sparse_attn_prefill_paged(const void *Q, const void *K_pages, const void *V_pages,
                                         const int32_t *block_table, const int32_t *q_pos, const int32_t *idx,
                                         void *O, float *lse, int B, int Hq, int Hkv, int Tq, int max_blocks,
                                         int num_pages, int d, int topk, float sm_scale, qsa_stream_t stream)
{
    const char *name = "qsa_sparse_attn_prefill_paged";
    if (!Q || !K_pages || !V_pages || !block_table || !q_pos || !idx || !O)
        return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Hq % Hkv || max_blocks <= 0 || num_pages <= 0 ||
        (long)Tq > 64L * max_blocks)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if ((long)num_pages * Hkv * 64 >= (1L << 31) || (long)max_blocks * 64 >= (1L << 31) ||
        (long)B * Tq >= (1L << 31))
        return fail(QSA_ERR_UNSUPPORTED, "%s: too large", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d", name, G);
    if (!aligned16(Q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(idx) || !aligned16(O) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) || (reinterpret_cast<uintptr_t>(block_table) & 3) ||
        (reinterpret_cast<uintptr_t>(q_pos) & 3))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    Paging pg;
    pg.q_pos = q_pos;
    pg.block_table = block_table;
    pg.max_blocks = max_blocks;
    pg.num_pages = num_pages;
    const int T = 64 * max_blocks;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 128 && G == 8) return launch_prefill<128, 8>(Q, K_pages, V_pages, idx, O, lse, B, Hq, Hkv, Tq, 0, T, topk, sm_scale, s, pg);
    if (d == 128 && G == 4) return launch_prefill<128, 4>(Q, K_pages, V_pages, idx, O, lse, B, Hq, Hkv, Tq, 0, T, topk, sm_scale, s, pg);
    if (d == 64 && G == 8) return launch_prefill<64, 8>(Q, K_pages, V_pages, idx, O, lse, B, Hq, Hkv, Tq, 0, T, topk, sm_scale, s, pg);
    return launch_prefill<64, 4>(Q, K_pages, V_pages, idx, O, lse, B, Hq, Hkv, Tq, 0, T, topk, sm_scale, s, pg);
}

qsa_status qsa_decode_paged(const void *q, const void *K_pages, const void *V_pages, const int32_t *block_table,
                            const int32_t *seq_lens, const int32_t *idx, void *o, int B, int Hq, int Hkv,
                            int max_blocks, int num_pages, int d, int topk, float sm_scale, qsa_stream_t stream)
{
    const char *name = "qsa_decode_paged";
    if (!q || !K_pages || !V_pages || !block_table || !seq_lens || !idx || !o)
        return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || max_blocks <= 0 || num_pages <= 0)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if ((long)num_pages * Hkv * 64 >= (1L << 31) || (long)max_blocks * 64 >= (1L << 31))
        return fail(QSA_ERR_UNSUPPORTED, "%s: cache too large", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d", name, G);
    if (!aligned16(q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(idx) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3) || (reinterpret_cast<uintptr_t>(seq_lens) & 3))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    if (B * Hkv > 65535) return fail(QSA_ERR_UNSUPPORTED, "%s: more than 65535 (sequence, group) rows", name);
    Paging pg;
    pg.seq_lens = seq_lens;
    pg.block_table = block_table;
    pg.max_blocks = max_blocks;
    pg.num_pages = num_pages;
    const int T = 64 * max_blocks;   // the kernel takes each sequence's length from seq_lens
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 128 && G == 8) return launch_decode<128, 8>(q, K_pages, V_pages, idx, o, B, Hq, Hkv, T, T, topk, sm_scale, s, pg);
    if (d == 128 && G == 4) return launch_decode<128, 4>(q, K_pages, V_pages, idx, o, B, Hq, Hkv, T, T, topk, sm_scale, s, pg);
    if (d == 64 && G == 8) return launch_decode<64, 8>(q, K_pages, V_pages, idx, o, B, Hq, Hkv, T, T, topk, sm_scale, s, pg);
    return launch_decode<64, 4>(q, K_pages, V_pages, idx, o, B, Hq, Hkv, T, T, topk, sm_scale, s, pg);
}

qsa_status qsa_quantize_kv_fp8(const void *X, void *codes, float *scales, int64_t rows, int d,
                               qsa_stream_t stream)
{
    if (!X || !codes || !scales) return fail(QSA_ERR_INVALID_ARG, "qsa_quantize_kv_fp8: null pointer");
    if (rows < 0) return fail(QSA_ERR_INVALID_ARG, "qsa_quantize_kv_fp8: rows=%lld", (long long)rows);
    if (d != 128) return fail(QSA_ERR_UNSUPPORTED, "qsa_quantize_kv_fp8: d=%d (rotated fp8 rows are 128 wide)", d);
    if (!aligned16(X) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3))
        return fail(QSA_ERR_INVALID_ARG, "qsa_quantize_kv_fp8: misaligned pointer");
    if (rows == 0) return QSA_OK;
    const long blocks = (rows + 7) / 8;   // 8 rows (warps) per CTA
    if (blocks >= (1L << 31)) return fail(QSA_ERR_UNSUPPORTED, "qsa_quantize_kv_fp8: too many rows");
    qsa::quantize_kv_fp8_kernel<128><<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(X), static_cast<uint8_t *>(codes), scales, (long)rows);
    return launched("quantize_kv_fp8_kernel");
}

qsa_status qsa_decode_fp8(const void *q, const void *K_codes, const float *K_scales, const void *V_codes,
                          const float *V_scales, const int32_t *idx, void *o, int B, int Hq, int Hkv, int L,
                          int T_kv_max, int d, int topk, float sm_scale, qsa_stream_t stream)
{
    const char *name = "qsa_decode_fp8";
    if (!q || !K_codes || !K_scales || !V_codes || !V_scales || !idx || !o)
        return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || T_kv_max <= 0 || T_kv_max % 64 || L > T_kv_max || Hq % Hkv)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if ((long)B * Hkv * T_kv_max >= (1L << 31)) return fail(QSA_ERR_UNSUPPORTED, "%s: cache too large", name);
    if (d != 128) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d (rotated fp8 rows are 128 wide)", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d", name, G);
    if (!aligned16(q) || !aligned16(K_codes) || !aligned16(V_codes) || !aligned16(K_scales) ||
        !aligned16(V_scales) || !aligned16(idx) || !aligned16(o))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    if (B * Hkv > 65535) return fail(QSA_ERR_UNSUPPORTED, "%s: more than 65535 (sequence, group) rows", name);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (G == 8)
        return launch_decode<128, 8, true>(q, K_codes, V_codes, idx, o, B, Hq, Hkv, L, T_kv_max, topk, sm_scale, s,
                                           Paging(), K_scales, V_scales);
    return launch_decode<128, 4, true>(q, K_codes, V_codes, idx, o, B, Hq, Hkv, L, T_kv_max, topk, sm_scale, s,
                                       Paging(), K_scales, V_scales);
}

qsa_status qsa_decode_fp8_paged(const void *q, const void *K_codes, const float *K_scales, const void *V_codes,
                                const float *V_scales, const int32_t *block_table, const int32_t *seq_lens,
                                const int32_t *idx, void *o, int B, int Hq, int Hkv, int max_blocks, int num_pages,
                                int d, int topk, float sm_scale, qsa_stream_t stream)
{
    const char *name = "qsa_decode_fp8_paged";
    if (!q || !K_codes || !K_scales || !V_codes || !V_scales || !block_table || !seq_lens || !idx || !o)
        return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || max_blocks <= 0 || num_pages <= 0)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if ((long)num_pages * Hkv * 64 >= (1L << 31) || (long)max_blocks * 64 >= (1L << 31))
        return fail(QSA_ERR_UNSUPPORTED, "%s: cache too large", name);
    if (d != 128) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d (rotated fp8 rows are 128 wide)", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d", name, G);
    if (!aligned16(q) || !aligned16(K_codes) || !aligned16(V_codes) || !aligned16(K_scales) ||
        !aligned16(V_scales) || !aligned16(idx) || !aligned16(o) || (reinterpret_cast<uintptr_t>(block_table) & 3) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    if (B * Hkv > 65535) return fail(QSA_ERR_UNSUPPORTED, "%s: more than 65535 (sequence, group) rows", name);
    Paging pg;
    pg.seq_lens = seq_lens;
    pg.block_table = block_table;
    pg.max_blocks = max_blocks;
    pg.num_pages = num_pages;
    const int T = 64 * max_blocks;   // the kernel takes each sequence's length from seq_lens
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (G == 8)
        return launch_decode<128, 8, true>(q, K_codes, V_codes, idx, o, B, Hq, Hkv, T, T, topk, sm_scale, s, pg,
                                           K_scales, V_scales);
    return launch_decode<128, 4, true>(q, K_codes, V_codes, idx, o, B, Hq, Hkv, T, T, topk, sm_scale, s, pg,
                                       K_scales, V_scales);
}

// ------------------------------------------------------ sharded caches
namespace {
// Candidates of the rows of a chunk at q_pos0 .. q_pos0 + Tq - 1 that lie in
// [blk_lo, blk_hi): their count for the longest row, and their first block.
void local_candidates(int Tq, int q_pos0, int blk_lo, int blk_hi, int &first, int &count)
{
    const int Dmax = (q_pos0 + Tq - 1) / 64;
    first = blk_lo > 1 ? blk_lo : 1;
    const int last = (Dmax - 1 < blk_hi - 1) ? Dmax - 1 : blk_hi - 1;
    count = last >= first ? last - first + 1 : 0;
}
constexpr int kLocalCH = 2048;
}  // namespace

int qsa_select_local_lists(int Tq, int q_pos0, int blk_lo, int blk_hi)
{
    if (Tq <= 0 || q_pos0 < 0 || blk_lo < 0 || blk_hi < blk_lo) return 0;
    int first, count;
    local_candidates(Tq, q_pos0, blk_lo, blk_hi, first, count);
    return count > 0 ? (count + kLocalCH - 1) / kLocalCH : 1;
}

size_t qsa_score_select_local_workspace(int B, int Hq, int Hkv, int Tq, int q_pos0, int d, int blk_lo, int blk_hi)
{
    (void)Hq;
    if (B <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || !supported_d(d) || blk_lo < 0 || blk_hi < blk_lo) return 0;
    int first, count;
    local_candidates(Tq, q_pos0, blk_lo, blk_hi, first, count);
    const size_t rows = (size_t)B * Hkv * ((Tq + 63) / 64);
    return align256(rows * d * sizeof(float)) + align256(rows * (size_t)((count + 3) / 4 * 4) * sizeof(float));
}

qsa_status qsa_score_select_local(const void *Q, const float *Kc_local, uint64_t *lists, int B, int Hq, int Hkv,
                                  int Tq, int q_pos0, int blk_lo, int blk_hi, int nlists, int d, int topk,
                                  float sm_scale, void *workspace, size_t workspace_bytes, qsa_stream_t stream)
{
    const char *name = "qsa_score_select_local";
    if (!Q || !Kc_local || !lists) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || q_pos0 % 64 || Hq % Hkv || blk_lo < 0 ||
        blk_hi <= blk_lo)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape or block range", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    if ((long)Hq * d / 8 > 1024) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq*d too large", name);
    const int need_lists = qsa_select_local_lists(Tq, q_pos0, blk_lo, blk_hi);
    if (nlists < need_lists || nlists > 64)
        return fail(QSA_ERR_INVALID_ARG, "%s: nlists=%d (this range needs %d, at most 64)", name, nlists, need_lists);
    if (!aligned16(Q) || !aligned16(Kc_local) || !aligned16(lists) || (workspace && !aligned16(workspace)))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    const size_t need = qsa_score_select_local_workspace(B, Hq, Hkv, Tq, q_pos0, d, blk_lo, blk_hi);
    if (!workspace || workspace_bytes < need)
        return fail(QSA_ERR_WORKSPACE, "%s: workspace needs %zu bytes", name, need);
    int first, count;
    local_candidates(Tq, q_pos0, blk_lo, blk_hi, first, count);
    const int NR = (Tq + 63) / 64;
    const size_t rows = (size_t)B * Hkv * NR;
    float *Qbar = static_cast<float *>(workspace);
    float *table = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + align256(rows * d * sizeof(float)));
    const int TS = (count + 3) / 4 * 4;
    const int nblk_max = (q_pos0 + Tq + 63) / 64;    // positions of the chunk bound every row's diagonal
    const int kc_n = blk_hi - blk_lo;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const dim3 pgrid(NR, B);
    const PoolLaunch pl = plan_pool(Hq, d, 64, (long)NR * B);
    const TableLaunch tl = plan_table(B, Hkv, Tq, q_pos0, first, blk_hi, d);
    qsa_status st;
    if (d == 128) {
        if ((st = set_smem(qsa::pool_queries_kernel<128>, pl.smem)) != QSA_OK) return st;
        qsa::pool_queries_kernel<128><<<pgrid, pl.threads, pl.smem, s>>>((const __nv_bfloat16 *)Q, Qbar, Tq, Hq, Hkv,
                                                                         64, pl.TS);
        if ((st = launched("pool_queries_kernel")) != QSA_OK) return st;
        if (count > 0) {
            if ((st = set_smem(qsa::score_table_kernel<128, float>, tl.smem)) != QSA_OK) return st;
            qsa::score_table_kernel<128, float><<<tl.grid, 256, tl.smem, s>>>(Qbar, Kc_local, table, nblk_max, Tq,
                                                                              q_pos0, TS, sm_scale, Hkv, nullptr, first,
                                                                              blk_hi, blk_lo, kc_n, first);
            if ((st = launched("score_table_kernel")) != QSA_OK) return st;
        }
    } else {
        if ((st = set_smem(qsa::pool_queries_kernel<64>, pl.smem)) != QSA_OK) return st;
        qsa::pool_queries_kernel<64><<<pgrid, pl.threads, pl.smem, s>>>((const __nv_bfloat16 *)Q, Qbar, Tq, Hq, Hkv,
                                                                        64, pl.TS);
        if ((st = launched("pool_queries_kernel")) != QSA_OK) return st;
        if (count > 0) {
            if ((st = set_smem(qsa::score_table_kernel<64, float>, tl.smem)) != QSA_OK) return st;
            qsa::score_table_kernel<64, float><<<tl.grid, 256, tl.smem, s>>>(Qbar, Kc_local, table, nblk_max, Tq,
                                                                             q_pos0, TS, sm_scale, Hkv, nullptr, first,
                                                                             blk_hi, blk_lo, kc_n, first);
            if ((st = launched("score_table_kernel")) != QSA_OK) return st;
        }
    }
    const int ssmem = kLocalCH * 8;
    if ((st = set_smem(qsa::local_lists_kernel, ssmem)) != QSA_OK) return st;
    qsa::local_lists_kernel<<<dim3(nlists, NR, B * Hkv), qsa::kSelThreads, ssmem, s>>>(
        table, lists, nblk_max, Tq, q_pos0, topk, kLocalCH, nlists, Hkv, first, blk_hi, TS);
    return launched("local_lists_kernel");
}

qsa_status qsa_merge_select_lists(const uint64_t *lists, int32_t *idx, int B, int Hkv, int Tq, int q_pos0,
                                  int nranks, int nlists, int topk, qsa_stream_t stream)
{
    const char *name = "qsa_merge_select_lists";
    if (!lists || !idx) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || q_pos0 % 64 || nlists <= 0 || nranks <= 0)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    if ((long)nranks * nlists * qsa::kMaxChosen * 8 > 200 * 1024)
        return fail(QSA_ERR_UNSUPPORTED, "%s: too many lists", name);
    if (!aligned16(lists) || !aligned16(idx)) return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    const int NR = (Tq + 63) / 64;
    const int msmem = nranks * nlists * qsa::kMaxChosen * 8;
    qsa_status st;
    if ((st = set_smem(qsa::merge_lists_kernel, msmem)) != QSA_OK) return st;
    qsa::merge_lists_kernel<<<dim3(NR, B * Hkv), qsa::kSelThreads, msmem, reinterpret_cast<cudaStream_t>(stream)>>>(
        lists, idx, Tq, q_pos0, topk, nlists, nranks);
    return launched("merge_lists_kernel");
}

qsa_status qsa_sparse_attn_prefill_local(const void *Q, const void *K_local, const void *V_local, const int32_t *idx,
                                         void *O, float *lse, int B, int Hq, int Hkv, int Tq, int q_pos0, int T_local,
                                         int blk_lo, int blk_hi, int d, int topk, float sm_scale, qsa_stream_t stream)
{
    const char *name = "qsa_sparse_attn_prefill_local";
    if (!Q || !K_local || !V_local || !idx || !O || !lse) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || q_pos0 % 64 || T_local <= 0 || T_local % 64 ||
        Hq % Hkv || blk_lo < 0 || blk_hi <= blk_lo || (long)(blk_hi - blk_lo) * 64 > T_local)
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape or block range", name);
    if ((long)B * Hkv * T_local >= (1L << 31) || (long)B * Tq >= (1L << 31))
        return fail(QSA_ERR_UNSUPPORTED, "%s: tensor too large", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if (topk < 2 || topk > 64) return fail(QSA_ERR_UNSUPPORTED, "%s: topk=%d", name, topk);
    const int G = Hq / Hkv;
    if (G != 4 && G != 8) return fail(QSA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d", name, G);
    if (!aligned16(Q) || !aligned16(K_local) || !aligned16(V_local) || !aligned16(idx) || !aligned16(O) ||
        (reinterpret_cast<uintptr_t>(lse) & 3))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Ownership own;
    own.lo = blk_lo;
    own.hi = blk_hi;
    own.partial = 1;
    const Paging pg;
    if (d == 128 && G == 8)
        return launch_prefill<128, 8>(Q, K_local, V_local, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_local, topk, sm_scale,
                                      s, pg, own);
    if (d == 128 && G == 4)
        return launch_prefill<128, 4>(Q, K_local, V_local, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_local, topk, sm_scale,
                                      s, pg, own);
    if (d == 64 && G == 8)
        return launch_prefill<64, 8>(Q, K_local, V_local, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_local, topk, sm_scale,
                                     s, pg, own);
    return launch_prefill<64, 4>(Q, K_local, V_local, idx, O, lse, B, Hq, Hkv, Tq, q_pos0, T_local, topk, sm_scale, s,
                                 pg, own);
}

qsa_status qsa_merge_partials(const void *O_parts, const float *lse_parts, void *O, float *lse, int nparts,
                              int64_t rows, int d, qsa_stream_t stream)
{
    const char *name = "qsa_merge_partials";
    if (!O_parts || !lse_parts || !O) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    if (nparts <= 0 || rows < 0) return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    if (!supported_d(d)) return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d", name, d);
    if ((reinterpret_cast<uintptr_t>(O_parts) & 15) || (reinterpret_cast<uintptr_t>(O) & 15) ||
        (reinterpret_cast<uintptr_t>(lse_parts) & 3) || (reinterpret_cast<uintptr_t>(lse) & 3))
        return fail(QSA_ERR_INVALID_ARG, "%s: misaligned pointer", name);
    if (rows == 0) return QSA_OK;
    const long per_cta = 8L * (256 / d);   // 8 warps, 256 / d rows per warp
    if ((rows + per_cta - 1) / per_cta >= (1L << 31)) return fail(QSA_ERR_UNSUPPORTED, "%s: too many rows", name);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
    if (d == 128)
        qsa::merge_partials_kernel<128><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)O_parts, lse_parts,
                                                             (__nv_bfloat16 *)O, lse, nparts, rows);
    else
        qsa::merge_partials_kernel<64><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)O_parts, lse_parts,
                                                            (__nv_bfloat16 *)O, lse, nparts, rows);
    return launched("merge_partials_kernel");
}

qsa_status qsa_prefill_pipeline_create(qsa_prefill_pipeline **out, int B, int Hq, int Hkv, int Tq, int q_pos0,
                                       int T_kv_max, int d, int topk, float sm_scale)
{
    const char *name = "qsa_prefill_pipeline_create";
    if (!out) return fail(QSA_ERR_INVALID_ARG, "%s: null out", name);
    *out = nullptr;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || q_pos0 < 0 || T_kv_max <= 0 || Hq % Hkv != 0 ||
        (T_kv_max & 63) || (q_pos0 & 63) || (long)q_pos0 + Tq > T_kv_max || !(sm_scale > 0.f))
        return fail(QSA_ERR_INVALID_ARG, "%s: bad shape", name);
    const int G = Hq / Hkv;
    if (!supported_d(d) || (G != 4 && G != 8) || topk < 2 || topk > 64)
        return fail(QSA_ERR_UNSUPPORTED, "%s: d=%d G=%d topk=%d", name, d, G, topk);
    auto *p = new (std::nothrow) qsa_prefill_pipeline;   // no exception crosses the C ABI
    if (!p) return fail(QSA_ERR_CUDA, "%s: host allocation failed", name);
    p->B = B, p->Hq = Hq, p->Hkv = Hkv, p->Tq = Tq, p->q_pos0 = q_pos0, p->T_kv_max = T_kv_max, p->d = d;
    p->topk = topk, p->sm_scale = sm_scale;
    const int NR = (Tq + 63) / 64;
    p->q_bytes = (size_t)B * Tq * Hq * d * 2;
    p->kv_bytes = (size_t)B * Hkv * T_kv_max * d * 2;
    p->kc_bytes = (size_t)B * Hkv * (T_kv_max / 64) * d * 4;
    p->idx_bytes = (size_t)B * Hkv * NR * topk * 4;
    p->ws_bytes = qsa_score_select_workspace(B, Hq, Hkv, Tq, q_pos0, 64, d, topk);
    cudaError_t e = cudaSuccess;
    auto chk = [&](cudaError_t r) {
        if (e == cudaSuccess) e = r;
    };
    chk(cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking));
    chk(cudaStreamCreateWithFlags(&p->s_cmp, cudaStreamNonBlocking));
    chk(cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking));
    for (auto &x : p->set) {
        chk(cudaMalloc(&x.Q, p->q_bytes));
        chk(cudaMalloc(&x.O, p->q_bytes));
        chk(cudaMalloc(&x.K, p->kv_bytes));
        chk(cudaMalloc(&x.V, p->kv_bytes));
        chk(cudaMalloc(reinterpret_cast<void **>(&x.Kc), p->kc_bytes));
        chk(cudaMalloc(reinterpret_cast<void **>(&x.idx), p->idx_bytes));
        if (p->ws_bytes) chk(cudaMalloc(&x.ws, p->ws_bytes));
        if (e == cudaSuccess) chk(cudaMemsetAsync(x.Kc, 0, p->kc_bytes, p->s_cmp));
        chk(cudaEventCreateWithFlags(&x.up, cudaEventDisableTiming));
        chk(cudaEventCreateWithFlags(&x.done, cudaEventDisableTiming));
        chk(cudaEventCreateWithFlags(&x.down, cudaEventDisableTiming));
    }
    if (e != cudaSuccess) {
        pipeline_free(p);
        return fail(QSA_ERR_CUDA, "%s: %s", name, cudaGetErrorString(e));
    }
    *out = p;
    return QSA_OK;
}

qsa_status qsa_prefill_pipeline_submit(qsa_prefill_pipeline *p, const void *hQ, const void *hK, const void *hV,
                                       void *hO)
{
    const char *name = "qsa_prefill_pipeline_submit";
    if (!p || !hQ || !hK || !hV || !hO) return fail(QSA_ERR_INVALID_ARG, "%s: null pointer", name);
    auto &x = p->set[p->k & 1];
    cudaError_t e = cudaSuccess;
    auto chk = [&](cudaError_t r) {
        if (e == cudaSuccess) e = r;
    };
    // upload: once step k-2's compute has read this set's inputs
    if (x.used) chk(cudaStreamWaitEvent(p->s_in, x.done, 0));
    chk(cudaMemcpyAsync(x.Q, hQ, p->q_bytes, cudaMemcpyHostToDevice, p->s_in));
    chk(cudaMemcpyAsync(x.K, hK, p->kv_bytes, cudaMemcpyHostToDevice, p->s_in));
    chk(cudaMemcpyAsync(x.V, hV, p->kv_bytes, cudaMemcpyHostToDevice, p->s_in));
    chk(cudaEventRecord(x.up, p->s_in));
    // compute: once the upload is in and step k-2's O has been read out
    chk(cudaStreamWaitEvent(p->s_cmp, x.up, 0));
    if (x.used) chk(cudaStreamWaitEvent(p->s_cmp, x.down, 0));
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "%s: %s", name, cudaGetErrorString(e));
    qsa_stream_t sc = reinterpret_cast<qsa_stream_t>(p->s_cmp);
    qsa_status st = qsa_compress_keys(x.K, x.Kc, p->B, p->Hkv, p->T_kv_max, p->d, 0, (p->q_pos0 + p->Tq) / 64, sc);
    if (st == QSA_OK)
        st = qsa_score_select(x.Q, x.Kc, x.idx, p->B, p->Hq, p->Hkv, p->Tq, p->q_pos0, 64, p->T_kv_max, p->d,
                              p->topk, p->sm_scale, x.ws, p->ws_bytes, sc);
    if (st == QSA_OK)
        st = qsa_sparse_attn_prefill(x.Q, x.K, x.V, x.idx, x.O, nullptr, p->B, p->Hq, p->Hkv, p->Tq, p->q_pos0,
                                     p->T_kv_max, p->d, p->topk, p->sm_scale, sc);
    if (st != QSA_OK) return st;
    chk(cudaEventRecord(x.done, p->s_cmp));
    // download: once the step's compute is done
    chk(cudaStreamWaitEvent(p->s_out, x.done, 0));
    chk(cudaMemcpyAsync(hO, x.O, p->q_bytes, cudaMemcpyDeviceToHost, p->s_out));
    chk(cudaEventRecord(x.down, p->s_out));
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "%s: %s", name, cudaGetErrorString(e));
    x.used = true;
    p->k++;
    return QSA_OK;
}

qsa_status qsa_prefill_pipeline_synchronize(qsa_prefill_pipeline *p)
{
    if (!p) return fail(QSA_ERR_INVALID_ARG, "qsa_prefill_pipeline_synchronize: null pipeline");
    for (cudaStream_t s : {p->s_in, p->s_cmp, p->s_out}) {
        const cudaError_t e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "qsa_prefill_pipeline_synchronize: %s", cudaGetErrorString(e));
    }
    return QSA_OK;
}

qsa_status qsa_prefill_pipeline_streams(qsa_prefill_pipeline *p, qsa_stream_t *copy_in, qsa_stream_t *compute,
                                        qsa_stream_t *copy_out)
{
    if (!p) return fail(QSA_ERR_INVALID_ARG, "qsa_prefill_pipeline_streams: null pipeline");
    if (copy_in) *copy_in = reinterpret_cast<qsa_stream_t>(p->s_in);
    if (compute) *compute = reinterpret_cast<qsa_stream_t>(p->s_cmp);
    if (copy_out) *copy_out = reinterpret_cast<qsa_stream_t>(p->s_out);
    return QSA_OK;
}

qsa_status qsa_prefill_pipeline_destroy(qsa_prefill_pipeline *p)
{
    pipeline_free(p);
    return QSA_OK;
}

qsa_status qsa_get_device_status(qsa_stream_t stream, int *detail)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return check_launch("cudaStreamSynchronize");
    int code = 0, det = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&code, qsa::g_status, sizeof(int)) != cudaSuccess ||
        cudaMemcpyFromSymbol(&det, qsa::g_status_detail, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(qsa::g_status, &zero, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(qsa::g_status_detail, &zero, sizeof(int)) != cudaSuccess)
        return check_launch("status word");
    if (detail) *detail = det;
    return (qsa_status)code;
}

qsa_status qsa_selftest_wait_timeout(uint64_t timeout_ns, qsa_stream_t stream)
{
    if (timeout_ns == 0 || timeout_ns > 1000000000ull)
        return fail(QSA_ERR_INVALID_ARG, "qsa_selftest_wait_timeout: limit must be in (0, 1 s]");
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return launched("selftest_wait_kernel");
}

qsa_status qsa_selftest_exp2(const float *x, float *y, int n, qsa_stream_t stream)
{
    if (!x || !y || n < 0) return fail(QSA_ERR_INVALID_ARG, "qsa_selftest_exp2: bad arguments");
    if (n == 0) return QSA_OK;
    const int pairs = (n + 1) / 2;
    selftest_exp2_kernel<false><<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    return launched("selftest_exp2_kernel");
}

qsa_status qsa_selftest_exp2_weight(const float *x, float *y, int n, qsa_stream_t stream)
{
    if (!x || !y || n < 0) return fail(QSA_ERR_INVALID_ARG, "qsa_selftest_exp2_weight: bad arguments");
    if (n == 0) return QSA_OK;
    const int pairs = (n + 1) / 2;
    selftest_exp2_kernel<true><<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    return launched("selftest_exp2_kernel");
}

const char *qsa_status_string(qsa_status s)
{
    switch (s) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
    case QSA_ERR_TIMEOUT: return "QSA_ERR_TIMEOUT";
    case QSA_ERR_BOUNDS: return "QSA_ERR_BOUNDS";
    case QSA_ERR_WORKSPACE: return "QSA_ERR_WORKSPACE";
    }
    return "QSA_ERR_UNKNOWN";
}

const char *qsa_last_error(void) { return g_last_error; }

unsigned long long qsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
