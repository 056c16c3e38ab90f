"""B200-native Qwen Sparse Attention (QSA) hot path.

Thin ctypes binding over ``libqsa.so`` (C ABI in ``include/qsa.h``).  Every
step of the path runs in the library's sm_100a kernels; this module only
checks tensor metadata and passes pointers, sizes and the current CUDA
stream.  PyTorch supplies device memory and streams.  There is no CPU or
PyTorch fallback: if the library is missing, importing this package raises.

Steps (pages "Qwen4 architecture: QSA, GR, PLE", section "1. QSA: not
looking at every token equally"; "Qwen4 in llama.cpp: Dissecting PR
#27742", section "QSA Is an Address-Selection Problem, Not a New Attention
Equation"):
    compress_keys        mean-pooled 64-token key summaries (fp32)
    score_select         pooled-query fp32 block scores -> top-k block ids
    sparse_attn_prefill  tcgen05/TMEM attention over the selected blocks
    decode               split-K single-token attention over the selected blocks
"""
import ctypes
import os
import re

import torch

BLOCK = 64
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "qsa.h")

# Size of the static scratch buffer of qsa_score_select_noalloc
# (QSA_SELECT_SCRATCH_BYTES in include/qsa.h).
SELECT_SCRATCH_BYTES = 4 << 20

STATUS = {0: "QSA_OK", 1: "QSA_ERR_INVALID_ARG", 2: "QSA_ERR_UNSUPPORTED", 3: "QSA_ERR_CUDA",
          4: "QSA_ERR_TIMEOUT", 5: "QSA_ERR_BOUNDS", 6: "QSA_ERR_WORKSPACE"}


class QSAError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with "
            "`python block_sparse_long_compress_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    sig = {
        "qsa_compress_keys": (I, [P, P, I, I, I, I, I, I, P]),
        "qsa_compress_keys_bf16": (I, [P, P, I, I, I, I, I, I, P]),
        "qsa_score_select_workspace": (S, [I, I, I, I, I, I, I, I]),
        "qsa_score_select": (I, [P, P, P, I, I, I, I, I, I, I, I, I, F, P, S, P]),
        "qsa_score_select_bf16": (I, [P, P, P, I, I, I, I, I, I, I, I, I, F, P, S, P]),
        "qsa_score_select_noalloc": (I, [P, P, P, I, I, I, I, I, I, I, I, I, F, P]),
        "qsa_sparse_attn_prefill": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P]),
        "qsa_decode_workspace": (S, [I, I, I, I, I]),
        "qsa_decode": (I, [P, P, P, P, P, I, I, I, I, I, I, I, F, P, S, P]),
        "qsa_compress_keys_paged": (I, [P, P, P, P, I, I, I, I, I, I, I, P]),
        "qsa_score_select_ragged": (I, [P, P, P, P, I, I, I, I, I, I, I, F, P]),
        "qsa_decode_paged": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]),
        "qsa_score_select_ragged_prefill": (I, [P, P, P, P, I, I, I, I, I, I, I, I, F, P, S, P]),
        "qsa_score_select_token_agg": (I, [P, P, P, P, I, I, I, I, I, I, I, I, F, I, P]),
        "qsa_score_select_prefill_agg_workspace": (S, [I, I, I, I, I, I, I, I, I]),
        "qsa_score_select_prefill_agg": (I, [P, P, P, I, I, I, I, I, I, I, I, F, I, P, S, P]),
        "qsa_quantize_kv_fp8": (I, [P, P, P, ctypes.c_int64, I, P]),
        "qsa_decode_fp8": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]),
        "qsa_decode_fp8_paged": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, P]),
        "qsa_sparse_attn_prefill_paged": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P]),
        "qsa_select_local_lists": (I, [I, I, I, I]),
        "qsa_score_select_local_workspace": (S, [I, I, I, I, I, I, I, I]),
        "qsa_score_select_local": (I, [P, P, P, I, I, I, I, I, I, I, I, I, I, F, P, S, P]),
        "qsa_merge_select_lists": (I, [P, P, I, I, I, I, I, I, I, P]),
        "qsa_sparse_attn_prefill_local": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, F, P]),
        "qsa_merge_partials": (I, [P, P, P, P, I, ctypes.c_int64, I, P]),
        "qsa_prefill_pipeline_create": (I, [ctypes.POINTER(P), I, I, I, I, I, I, I, I, F]),
        "qsa_prefill_pipeline_submit": (I, [P, P, P, P, P]),
        "qsa_prefill_pipeline_synchronize": (I, [P]),
        "qsa_prefill_pipeline_streams": (I, [P, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P)]),
        "qsa_prefill_pipeline_destroy": (I, [P]),
        "qsa_get_device_status": (I, [P, ctypes.POINTER(I)]),
        "qsa_selftest_wait_timeout": (I, [ctypes.c_uint64, P]),
        "qsa_selftest_exp2": (I, [P, P, I, P]),
        "qsa_selftest_exp2_weight": (I, [P, P, I, P]),
        "qsa_status_string": (ctypes.c_char_p, [I]),
        "qsa_last_error": (ctypes.c_char_p, []),
        "qsa_launch_count": (ctypes.c_ulonglong, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def lib():
    """The loaded ctypes library handle."""
    return _lib


def declared_symbols():
    """Entry points declared in include/qsa.h."""
    text = open(HEADER_PATH).read()
    return re.findall(r"QSA_API\s+[\w\s\*]+?\b(qsa_\w+)\s*\(", text)


def _check(rc, what):
    if rc != 0:
        msg = _lib.qsa_last_error().decode()
        raise QSAError(rc, f"{what} ({msg})" if msg else what)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t, dtype, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


# ------------------------------------------------------------------ steps
def _summary_fn(Kc, fp32_fn, bf16_fn):
    """The entry point for the summaries' dtype: fp32 (default) or bf16."""
    if isinstance(Kc, torch.Tensor) and Kc.dtype == torch.bfloat16:
        return bf16_fn, torch.bfloat16
    return fp32_fn, torch.float32


def compress_keys(K, Kc, blk_begin=0, blk_end=None, stream=None):
    """Kc[b,h,j,:] = mean of K[b,h,64j:64j+64,:] for j in [blk_begin, blk_end).
    K: bf16 [B, Hkv, T_kv_max, d]; Kc: fp32 [B, Hkv, T_kv_max//64, d], or bf16
    for the bf16-summary option (the fp32 mean rounded to nearest even)."""
    B, Hkv, T, d = K.shape
    if blk_end is None:
        blk_end = T // BLOCK
    if tuple(Kc.shape) != (B, Hkv, T // BLOCK, d):
        raise ValueError("Kc shape must be [B, Hkv, T_kv_max//64, d]")
    fn, kdt = _summary_fn(Kc, _lib.qsa_compress_keys, _lib.qsa_compress_keys_bf16)
    _check(fn(_ptr(K, torch.bfloat16, "K"), _ptr(Kc, kdt, "Kc"),
              B, Hkv, T, d, blk_begin, blk_end, _stream(stream)),
           fn.__name__)
    return Kc


def score_select_workspace(B, Hq, Hkv, Tq, q_pos0, qblk, d, topk):
    return int(_lib.qsa_score_select_workspace(B, Hq, Hkv, Tq, q_pos0, qblk, d, topk))


def score_select(Q, Kc, idx, topk, q_pos0, qblk=BLOCK, sm_scale=None, workspace=None,
                 stream=None):
    """Top-k block selection per (query block or token, KV group).
    Q: bf16 [B, Tq, Hq, d]; Kc: fp32 (or bf16) [B, Hkv, T_kv_max//64, d];
    idx: int32 [B, Hkv, ceil(Tq/qblk), topk] (written)."""
    B, Tq, Hq, d = Q.shape
    _, Hkv, nblk, _ = Kc.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    need = score_select_workspace(B, Hq, Hkv, Tq, q_pos0, qblk, d, topk)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    fn, kdt = _summary_fn(Kc, _lib.qsa_score_select, _lib.qsa_score_select_bf16)
    _check(fn(_ptr(Q, torch.bfloat16, "Q"), _ptr(Kc, kdt, "Kc"),
              _ptr(idx, torch.int32, "idx"), B, Hq, Hkv, Tq, q_pos0, qblk,
              nblk * BLOCK, d, topk, float(sm_scale),
              _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
              _stream(stream)),
           fn.__name__)
    return idx


def sparse_attn_prefill(Q, K, V, idx, O, q_pos0=0, sm_scale=None, lse=None, stream=None):
    """O = softmax attention of Q over the blocks in idx (keys <= position).
    Q, O: bf16 [B, Tq, Hq, d]; K, V: bf16 [B, Hkv, T_kv_max, d];
    idx: int32 [B, Hkv, ceil(Tq/64), topk]; lse: optional fp32 [B, Tq, Hq]."""
    B, Tq, Hq, d = Q.shape
    _, Hkv, T, _ = K.shape
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = d ** -0.5
    _check(_lib.qsa_sparse_attn_prefill(
        _ptr(Q, torch.bfloat16, "Q"), _ptr(K, torch.bfloat16, "K"), _ptr(V, torch.bfloat16, "V"),
        _ptr(idx, torch.int32, "idx"), _ptr(O, torch.bfloat16, "O"),
        _ptr(lse, torch.float32, "lse"), B, Hq, Hkv, Tq, q_pos0, T, d, topk, float(sm_scale),
        _stream(stream)), "qsa_sparse_attn_prefill")
    return O


def decode_workspace(B, Hq, Hkv, d, topk):
    return int(_lib.qsa_decode_workspace(B, Hq, Hkv, d, topk))


def decode(q, K, V, idx, o, L, sm_scale=None, workspace=None, stream=None):
    """Single-token attention per sequence over its selected blocks.
    q, o: bf16 [B, Hq, d] (or [B, 1, Hq, d]); K, V: bf16 [B, Hkv, T_kv_max, d];
    idx: int32 [B, Hkv, 1, topk]; L: cache length (query at position L-1)."""
    B, Hkv, T, d = K.shape
    Hq = q.shape[-2]
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = d ** -0.5
    need = decode_workspace(B, Hq, Hkv, d, topk)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(_lib.qsa_decode(
        _ptr(q, torch.bfloat16, "q"), _ptr(K, torch.bfloat16, "K"), _ptr(V, torch.bfloat16, "V"),
        _ptr(idx, torch.int32, "idx"), _ptr(o, torch.bfloat16, "o"), B, Hq, Hkv, L, T, d, topk,
        float(sm_scale), _ptr(workspace, torch.uint8, "workspace"),
        0 if workspace is None else workspace.numel(), _stream(stream)), "qsa_decode")
    return o


# ------------------------------------------------ ragged, paged caches
def compress_keys_paged(K_pages, block_table, seq_lens, Kc, blk_begin=0, blk_end=None, stream=None):
    """Summaries of the complete blocks among logical blocks [blk_begin,
    blk_end) of every sequence of a paged cache.  K_pages: bf16 [num_pages,
    Hkv, 64, d]; block_table: int32 [B, max_blocks]; seq_lens: int32 [B];
    Kc: fp32 [B, Hkv, max_blocks, d] (logical order)."""
    num_pages, Hkv, blk, d = K_pages.shape
    B, max_blocks = block_table.shape
    if blk != BLOCK or tuple(Kc.shape) != (B, Hkv, max_blocks, d):
        raise ValueError("K_pages must be [num_pages, Hkv, 64, d] and Kc [B, Hkv, max_blocks, d]")
    if blk_end is None:
        blk_end = max_blocks
    _check(_lib.qsa_compress_keys_paged(_ptr(K_pages, torch.bfloat16, "K_pages"),
                                        _ptr(block_table, torch.int32, "block_table"),
                                        _ptr(seq_lens, torch.int32, "seq_lens"),
                                        _ptr(Kc, torch.float32, "Kc"), B, Hkv, max_blocks, num_pages,
                                        d, blk_begin, blk_end, _stream(stream)),
           "qsa_compress_keys_paged")
    return Kc


def score_select_ragged(Q, Kc, seq_lens, idx, topk, max_len, sm_scale=None, stream=None):
    """Per-token selection for one token per sequence, each at position
    seq_lens[b] - 1.  Q: bf16 [B, 1, Hq, d]; Kc: fp32 [B, Hkv, max_blocks, d];
    idx: int32 [B, Hkv, 1, topk] (written); max_len >= every length."""
    B, _, Hq, d = Q.shape
    _, Hkv, max_blocks, _ = Kc.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    _check(_lib.qsa_score_select_ragged(_ptr(Q, torch.bfloat16, "Q"), _ptr(Kc, torch.float32, "Kc"),
                                        _ptr(seq_lens, torch.int32, "seq_lens"),
                                        _ptr(idx, torch.int32, "idx"), B, Hq, Hkv, max_blocks,
                                        int(max_len), d, topk, float(sm_scale), _stream(stream)),
           "qsa_score_select_ragged")
    return idx


def decode_paged(q, K_pages, V_pages, block_table, seq_lens, idx, o, sm_scale=None, stream=None):
    """Decode attention over the selected blocks of paged caches, each
    sequence at its own length.  q, o: bf16 [B, Hq, d]."""
    B, Hq, d = q.shape
    num_pages, Hkv, _, _ = K_pages.shape
    max_blocks = block_table.shape[1]
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = d ** -0.5
    _check(_lib.qsa_decode_paged(_ptr(q, torch.bfloat16, "q"), _ptr(K_pages, torch.bfloat16, "K_pages"),
                                 _ptr(V_pages, torch.bfloat16, "V_pages"),
                                 _ptr(block_table, torch.int32, "block_table"),
                                 _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(idx, torch.int32, "idx"),
                                 _ptr(o, torch.bfloat16, "o"), B, Hq, Hkv, max_blocks, num_pages, d,
                                 topk, float(sm_scale), _stream(stream)),
           "qsa_decode_paged")
    return o


AGGREGATORS = {"mean": 0, "max": 1, "softmax_sum": 2}


def score_select_token_agg(q, Kc, idx, topk, q_pos0, aggregator="mean", sm_scale=None, seq_lens=None,
                           stream=None):
    """Per-token selection with an aggregator of the group's per-head scores
    ("mean", "max" -- the same for one token --, or "softmax_sum").
    q: bf16 [B, Tq, Hq, d] at positions q_pos0 .. q_pos0 + Tq - 1, or with
    seq_lens (int32 [B], Tq = 1) at seq_lens[b] - 1 (q_pos0 = the largest);
    Kc fp32 [B, Hkv, max_blocks, d]; idx int32 [B, Hkv, Tq, topk] (written)."""
    if aggregator not in AGGREGATORS:
        raise ValueError(f"aggregator must be one of {sorted(AGGREGATORS)}, got {aggregator!r}")
    B, Tq, Hq, d = q.shape
    _, Hkv, max_blocks, _ = Kc.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    sl = None if seq_lens is None else _ptr(seq_lens, torch.int32, "seq_lens")
    _check(_lib.qsa_score_select_token_agg(_ptr(q, torch.bfloat16, "q"), _ptr(Kc, torch.float32, "Kc"), sl,
                                           _ptr(idx, torch.int32, "idx"), B, Hq, Hkv, Tq, q_pos0, max_blocks, d,
                                           topk, float(sm_scale), AGGREGATORS[aggregator], _stream(stream)),
           "qsa_score_select_token_agg")
    return idx


def score_select_prefill_agg_workspace(B, Hq, Hkv, Tq, q_pos0, T_kv_max, d, topk, aggregator):
    return int(_lib.qsa_score_select_prefill_agg_workspace(B, Hq, Hkv, Tq, q_pos0, T_kv_max, d, topk,
                                                          AGGREGATORS[aggregator]))


def score_select_prefill_agg(Q, Kc, idx, topk, q_pos0, aggregator="max", sm_scale=None, workspace=None,
                             stream=None):
    """Selection for 64-token query blocks under the max-over-tokens or the
    softmax-sum aggregator (per-(head, token) logits on the tensor cores).
    Q bf16 [B, Tq, Hq, 128]; Kc bf16 summaries [B, Hkv, T_kv_max//64, 128];
    idx int32 [B, Hkv, ceil(Tq/64), topk] (written)."""
    if aggregator not in ("max", "softmax_sum"):
        raise ValueError(f"prefill rows take the 'max' or 'softmax_sum' aggregator, got {aggregator!r} "
                         "(the mean is score_select over bf16 summaries)")
    B, Tq, Hq, d = Q.shape
    _, Hkv, nblk, _ = Kc.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    need = score_select_prefill_agg_workspace(B, Hq, Hkv, Tq, q_pos0, 64 * nblk, d, topk, aggregator)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=Q.device)
    _check(_lib.qsa_score_select_prefill_agg(_ptr(Q, torch.bfloat16, "Q"), _ptr(Kc, torch.bfloat16, "Kc"),
                                             _ptr(idx, torch.int32, "idx"), B, Hq, Hkv, Tq, q_pos0, 64 * nblk, d,
                                             topk, float(sm_scale), AGGREGATORS[aggregator],
                                             _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
                                             _stream(stream)),
           "qsa_score_select_prefill_agg")
    return idx


def score_select_ragged_prefill(Q, Kc, q_pos, idx, topk, max_pos, sm_scale=None, workspace=None,
                                stream=None):
    """Selection for a chunked prefill of a ragged batch: Q bf16 [B, Tq, Hq, d],
    sequence b's chunk at positions q_pos[b] .. q_pos[b] + Tq - 1 (int32 [B],
    multiples of 64); Kc fp32 [B, Hkv, max_blocks, d]; idx int32
    [B, Hkv, ceil(Tq/64), topk] (written); max_pos >= every q_pos[b]."""
    B, Tq, Hq, d = Q.shape
    _, Hkv, max_blocks, _ = Kc.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    need = score_select_workspace(B, Hq, Hkv, Tq, max_pos, BLOCK, d, topk)
    if workspace is None:
        workspace = torch.empty(max(1, need), dtype=torch.uint8, device=Q.device)
    _check(_lib.qsa_score_select_ragged_prefill(
        _ptr(Q, torch.bfloat16, "Q"), _ptr(Kc, torch.float32, "Kc"), _ptr(q_pos, torch.int32, "q_pos"),
        _ptr(idx, torch.int32, "idx"), B, Hq, Hkv, Tq, max_blocks, int(max_pos), d, topk, float(sm_scale),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "qsa_score_select_ragged_prefill")
    return idx


def sparse_attn_prefill_paged(Q, K_pages, V_pages, block_table, q_pos, idx, O, sm_scale=None, lse=None,
                              stream=None):
    """Prefill attention of a ragged batch over paged caches (each sequence's
    chunk at its own position q_pos[b]).  Q, O bf16 [B, Tq, Hq, d]."""
    B, Tq, Hq, d = Q.shape
    num_pages, Hkv, _, _ = K_pages.shape
    max_blocks = block_table.shape[1]
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = d ** -0.5
    _check(_lib.qsa_sparse_attn_prefill_paged(
        _ptr(Q, torch.bfloat16, "Q"), _ptr(K_pages, torch.bfloat16, "K_pages"),
        _ptr(V_pages, torch.bfloat16, "V_pages"), _ptr(block_table, torch.int32, "block_table"),
        _ptr(q_pos, torch.int32, "q_pos"), _ptr(idx, torch.int32, "idx"), _ptr(O, torch.bfloat16, "O"),
        _ptr(lse, torch.float32, "lse"), B, Hq, Hkv, Tq, max_blocks, num_pages, d, topk, float(sm_scale),
        _stream(stream)), "qsa_sparse_attn_prefill_paged")
    return O


# ------------------------------------------------- rotated fp8 KV (decode)
def quantize_kv_fp8(X, codes=None, scales=None, stream=None):
    """Rotated fp8 cache rows: X bf16 [..., 128] -> codes uint8 [..., 128]
    (e4m3 of the Walsh-Hadamard-rotated row over its scale) and scales fp32
    [...] (max |rotated row| / 448)."""
    if X.shape[-1] != 128:
        raise ValueError("rotated fp8 rows are 128 wide")
    if codes is None:
        codes = torch.empty(X.shape, dtype=torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty(X.shape[:-1], dtype=torch.float32, device=X.device)
    rows = X.numel() // 128
    _check(_lib.qsa_quantize_kv_fp8(_ptr(X, torch.bfloat16, "X"), _ptr(codes, torch.uint8, "codes"),
                                    _ptr(scales, torch.float32, "scales"), rows, 128, _stream(stream)),
           "qsa_quantize_kv_fp8")
    return codes, scales


def decode_fp8(q, K_codes, K_scales, V_codes, V_scales, idx, o, L, sm_scale=None, stream=None):
    """Decode attention over a rotated fp8 cache (codes uint8 [B, Hkv, T, 128],
    scales fp32 [B, Hkv, T]); q, o bf16 [B, Hq, 128] in the original basis."""
    B, Hq, d = q.shape
    _, Hkv, T, _ = K_codes.shape
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = d ** -0.5
    _check(_lib.qsa_decode_fp8(_ptr(q, torch.bfloat16, "q"), _ptr(K_codes, torch.uint8, "K_codes"),
                               _ptr(K_scales, torch.float32, "K_scales"), _ptr(V_codes, torch.uint8, "V_codes"),
                               _ptr(V_scales, torch.float32, "V_scales"), _ptr(idx, torch.int32, "idx"),
                               _ptr(o, torch.bfloat16, "o"), B, Hq, Hkv, L, T, d, topk, float(sm_scale),
                               _stream(stream)), "qsa_decode_fp8")
    return o


def decode_fp8_paged(q, K_codes, K_scales, V_codes, V_scales, block_table, seq_lens, idx, o, sm_scale=None,
                     stream=None):
    """Decode attention over paged rotated fp8 caches: codes uint8
    [num_pages, Hkv, 64, 128], scales fp32 [num_pages, Hkv, 64]; the rest as
    decode_paged."""
    B, Hq, d = q.shape
    num_pages, Hkv, _, _ = K_codes.shape
    max_blocks = block_table.shape[1]
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = d ** -0.5
    _check(_lib.qsa_decode_fp8_paged(_ptr(q, torch.bfloat16, "q"), _ptr(K_codes, torch.uint8, "K_codes"),
                                     _ptr(K_scales, torch.float32, "K_scales"),
                                     _ptr(V_codes, torch.uint8, "V_codes"), _ptr(V_scales, torch.float32, "V_scales"),
                                     _ptr(block_table, torch.int32, "block_table"),
                                     _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(idx, torch.int32, "idx"),
                                     _ptr(o, torch.bfloat16, "o"), B, Hq, Hkv, max_blocks, num_pages, d, topk,
                                     float(sm_scale), _stream(stream)), "qsa_decode_fp8_paged")
    return o


class QSADecodePaged:
    """The decode path for a ragged batch over paged caches: per-token
    selection at each sequence's own position, then split-K attention
    through the block table.  Summaries (logical order) are persistent
    state; compress() adds the blocks that have completed."""

    def __init__(self, B, Hq, Hkv, d, max_blocks, topk, device="cuda"):
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, d
        self.max_blocks, self.topk = max_blocks, topk
        self.sm_scale = d ** -0.5
        dev = torch.device(device)
        self.Kc = torch.zeros((B, Hkv, max_blocks, d), dtype=torch.float32, device=dev)
        self.idx = torch.empty((B, Hkv, 1, topk), dtype=torch.int32, device=dev)
        self.o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)

    def compress(self, K_pages, block_table, seq_lens, blk_begin=0, blk_end=None, stream=None):
        compress_keys_paged(K_pages, block_table, seq_lens, self.Kc, blk_begin, blk_end, stream)

    def __call__(self, q, K_pages, V_pages, block_table, seq_lens, max_len, stream=None):
        score_select_ragged(q.view(self.B, 1, self.Hq, self.d), self.Kc, seq_lens, self.idx, self.topk,
                            max_len, self.sm_scale, stream)
        decode_paged(q, K_pages, V_pages, block_table, seq_lens, self.idx, self.o, self.sm_scale,
                     stream)
        return self.o


# ----------------------------------- one sequence over several GPUs
def shard_ranges(n_blocks, world):
    """Contiguous block ranges [lo, hi) of a cache of n_blocks blocks split
    over `world` ranks, as equal as possible, in rank order."""
    if world <= 0 or n_blocks < world:
        raise ValueError("need at least one block per rank")
    base, extra = divmod(n_blocks, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def select_local_lists(Tq, q_pos0, blk_lo, blk_hi):
    """Lists per selection row a rank holding blocks [blk_lo, blk_hi) emits."""
    return int(_lib.qsa_select_local_lists(Tq, q_pos0, blk_lo, blk_hi))


def score_select_local_workspace(B, Hq, Hkv, Tq, q_pos0, d, blk_lo, blk_hi):
    return int(_lib.qsa_score_select_local_workspace(B, Hq, Hkv, Tq, q_pos0, d, blk_lo, blk_hi))


def score_select_local(Q, Kc_local, lists, q_pos0, blk_lo, blk_hi, topk, sm_scale=None, workspace=None,
                       stream=None):
    """A rank's candidate lists for prefill rows (64-token blocks) over its
    own blocks [blk_lo, blk_hi).  Q bf16 [B, Tq, Hq, d]; Kc_local fp32
    [B, Hkv, blk_hi - blk_lo, d]; lists int64 (uint64 keys) [B, Hkv, NR,
    nlists, 62] (written)."""
    B, Tq, Hq, d = Q.shape
    Hkv = Kc_local.shape[1]
    nlists = lists.shape[3]
    if sm_scale is None:
        sm_scale = d ** -0.5
    need = score_select_local_workspace(B, Hq, Hkv, Tq, q_pos0, d, blk_lo, blk_hi)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=Q.device)
    _check(_lib.qsa_score_select_local(_ptr(Q, torch.bfloat16, "Q"), _ptr(Kc_local, torch.float32, "Kc_local"),
                                       _ptr(lists, torch.int64, "lists"), B, Hq, Hkv, Tq, q_pos0, blk_lo, blk_hi,
                                       nlists, d, topk, float(sm_scale), _ptr(workspace, torch.uint8, "workspace"),
                                       workspace.numel(), _stream(stream)), "qsa_score_select_local")
    return lists


def merge_select_lists(lists, idx, Tq, q_pos0, stream=None):
    """Selection from all ranks' gathered lists ([R, B, Hkv, NR, nlists, 62]
    int64, rank-major) of a chunk of Tq tokens at q_pos0 into idx int32
    [B, Hkv, NR, topk]."""
    R, B, Hkv, NR, nlists, _ = lists.shape
    if NR != -(-Tq // BLOCK):
        raise ValueError("lists do not match Tq")
    topk = idx.shape[-1]
    _check(_lib.qsa_merge_select_lists(_ptr(lists, torch.int64, "lists"), _ptr(idx, torch.int32, "idx"), B, Hkv,
                                       Tq, q_pos0, R, nlists, topk, _stream(stream)), "qsa_merge_select_lists")
    return idx


def sparse_attn_prefill_local(Q, K_local, V_local, idx, O, lse, q_pos0, blk_lo, blk_hi, sm_scale=None, stream=None):
    """Attention over the listed blocks this rank holds ([blk_lo, blk_hi),
    block j at row 64 (j - blk_lo) of K_local / V_local bf16 [B, Hkv,
    T_local, d]); O bf16 [B, Tq, Hq, d] and lse fp32 [B, Tq, Hq] over the
    rank's keys (0 and -inf where it holds none of a row's blocks)."""
    B, Tq, Hq, d = Q.shape
    _, Hkv, T_local, _ = K_local.shape
    topk = idx.shape[-1]
    if sm_scale is None:
        sm_scale = d ** -0.5
    _check(_lib.qsa_sparse_attn_prefill_local(
        _ptr(Q, torch.bfloat16, "Q"), _ptr(K_local, torch.bfloat16, "K_local"),
        _ptr(V_local, torch.bfloat16, "V_local"), _ptr(idx, torch.int32, "idx"), _ptr(O, torch.bfloat16, "O"),
        _ptr(lse, torch.float32, "lse"), B, Hq, Hkv, Tq, q_pos0, T_local, blk_lo, blk_hi, d, topk,
        float(sm_scale), _stream(stream)), "qsa_sparse_attn_prefill_local")
    return O, lse


def merge_partials(O_parts, lse_parts, O, lse=None, stream=None):
    """O = sum_r exp(lse_r - L) O_r, L = logsumexp_r lse_r.  O_parts bf16
    [R, ..., d]; lse_parts fp32 [R, ...]; O bf16 [..., d]; lse fp32 [...]."""
    R = O_parts.shape[0]
    d = O_parts.shape[-1]
    rows = lse_parts[0].numel()
    _check(_lib.qsa_merge_partials(_ptr(O_parts, torch.bfloat16, "O_parts"), _ptr(lse_parts, torch.float32, "lse_parts"),
                                   _ptr(O, torch.bfloat16, "O"), _ptr(lse, torch.float32, "lse"), R, rows, d,
                                   _stream(stream)), "qsa_merge_partials")
    return O


def all_gather_rank_major(t, group=None):
    """[R, *t.shape]: every rank's tensor in rank order (a collective:
    every rank of the group calls it with a tensor of the same shape)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


class QSAShardedPrefill:
    """A chunked prefill of one sequence whose cache is split over the ranks
    of a process group (one GPU each): rank r holds the cache blocks
    blk_ranges[r] (contiguous, ascending in rank order; the last rank's range
    ends with the chunk's own blocks) with their summaries, and the whole Q.
    A step: the rank's candidate lists, an all-gather of the lists (a few
    KB), the merged selection (identical on every rank), attention over the
    rank's selected blocks, an all-gather of the partial outputs and their
    log-sum-exp merge.  Every rank gets the full output."""

    def __init__(self, B, Tq, Hq, Hkv, d, topk, q_pos0, blk_ranges, rank, group=None, device="cuda"):
        self.B, self.Tq, self.Hq, self.Hkv, self.d = B, Tq, Hq, Hkv, d
        self.topk, self.q_pos0, self.rank, self.group = topk, q_pos0, rank, group
        self.sm_scale = d ** -0.5
        self.blk_lo, self.blk_hi = blk_ranges[rank]
        self.nlists = max(select_local_lists(Tq, q_pos0, lo, hi) for lo, hi in blk_ranges)
        NR = -(-Tq // BLOCK)
        dev = torch.device(device)
        self.lists = torch.empty((B, Hkv, NR, self.nlists, 62), dtype=torch.int64, device=dev)
        self.ws = torch.empty(max(16, score_select_local_workspace(B, Hq, Hkv, Tq, q_pos0, d, self.blk_lo,
                                                                    self.blk_hi)), dtype=torch.uint8, device=dev)
        self.idx = torch.empty((B, Hkv, NR, topk), dtype=torch.int32, device=dev)
        self.O_part = torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=dev)
        self.lse_part = torch.empty((B, Tq, Hq), dtype=torch.float32, device=dev)
        self.O = torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=dev)

    def __call__(self, Q, K_local, V_local, Kc_local, stream=None):
        score_select_local(Q, Kc_local, self.lists, self.q_pos0, self.blk_lo, self.blk_hi, self.topk,
                           self.sm_scale, self.ws, stream)
        merge_select_lists(all_gather_rank_major(self.lists, self.group), self.idx, self.Tq, self.q_pos0, stream)
        sparse_attn_prefill_local(Q, K_local, V_local, self.idx, self.O_part, self.lse_part, self.q_pos0,
                                  self.blk_lo, self.blk_hi, self.sm_scale, stream)
        merge_partials(all_gather_rank_major(self.O_part, self.group),
                       all_gather_rank_major(self.lse_part, self.group), self.O, None, stream)
        return self.O


def device_status(stream=None):
    """Synchronise the stream; return (and clear) the kernels' status word."""
    det = ctypes.c_int(0)
    rc = _lib.qsa_get_device_status(_stream(stream), ctypes.byref(det))
    return STATUS.get(rc, rc), det.value


def selftest_wait_timeout(timeout_ns, stream=None):
    _check(_lib.qsa_selftest_wait_timeout(int(timeout_ns), _stream(stream)),
           "qsa_selftest_wait_timeout")


def launch_count():
    """Kernels launched by the library so far in this process."""
    return int(_lib.qsa_launch_count())


# --------------------------------------------------------------- pipeline
class QSAPrefill:
    """The whole prefill path for one shape: compress the new complete
    blocks, select, attend.  Owns its workspace, summaries and outputs
    (allocated once with torch)."""

    def __init__(self, B, Tq, Hq, Hkv, d, T_kv_max, topk, q_pos0=0, device="cuda",
                 with_lse=False, summary_dtype=torch.float32):
        self.B, self.Tq, self.Hq, self.Hkv, self.d = B, Tq, Hq, Hkv, d
        self.T_kv_max, self.topk, self.q_pos0 = T_kv_max, topk, q_pos0
        self.sm_scale = d ** -0.5
        NR = -(-Tq // BLOCK)
        dev = torch.device(device)
        self.Kc = torch.zeros((B, Hkv, T_kv_max // BLOCK, d), dtype=summary_dtype, device=dev)
        self.idx = torch.empty((B, Hkv, NR, topk), dtype=torch.int32, device=dev)
        self.O = torch.empty((B, Tq, Hq, d), dtype=torch.bfloat16, device=dev)
        self.lse = (torch.empty((B, Tq, Hq), dtype=torch.float32, device=dev)
                    if with_lse else None)
        self.ws = torch.empty(max(1, score_select_workspace(B, Hq, Hkv, Tq, q_pos0, BLOCK, d, topk)),
                              dtype=torch.uint8, device=dev)
        # blocks whose summaries this step must (re)compute: the complete
        # blocks that the new tokens finish
        self.blk_begin = q_pos0 // BLOCK
        self.blk_end = (q_pos0 + Tq) // BLOCK

    def precompress_cache(self, K, stream=None):
        """Summaries of the cache blocks before the new tokens (persistent state)."""
        if self.blk_begin > 0:
            compress_keys(K, self.Kc, 0, self.blk_begin, stream)

    def __call__(self, Q, K, V, stream=None):
        compress_keys(K, self.Kc, self.blk_begin, self.blk_end, stream)
        score_select(Q, self.Kc, self.idx, self.topk, self.q_pos0, BLOCK, self.sm_scale,
                     self.ws, stream)
        sparse_attn_prefill(Q, K, V, self.idx, self.O, self.q_pos0, self.sm_scale, self.lse,
                            stream)
        return self.O


class PrefillHostPipeline:
    """Prefill steps fed from pinned host memory: the library's native
    pipeline object (qsa_prefill_pipeline_*) owns two device buffer sets and
    three streams, so that step k's Q, K, V upload, step k-1's compute and
    step k-2's O download run at once.  This class only marshals arguments;
    s_in / s_out are the object's copy-in and copy-out streams (for timing
    events)."""

    def __init__(self, B, Tq, Hq, Hkv, d, T_kv_max, topk, q_pos0=0, device="cuda"):
        dev = torch.device(device)
        if dev.type != "cuda":
            raise ValueError("the pipeline runs on a CUDA device")
        self.shape_q = (B, Tq, Hq, d)
        self.shape_kv = (B, Hkv, T_kv_max, d)
        self._h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _check(_lib.qsa_prefill_pipeline_create(ctypes.byref(self._h), B, Hq, Hkv, Tq, q_pos0, T_kv_max, d,
                                                    topk, float(d ** -0.5)), "qsa_prefill_pipeline_create")
        sin, scmp, sout = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        _check(_lib.qsa_prefill_pipeline_streams(self._h, ctypes.byref(sin), ctypes.byref(scmp),
                                                 ctypes.byref(sout)), "qsa_prefill_pipeline_streams")
        self.s_in = torch.cuda.ExternalStream(sin.value, device=dev)
        self.s_cmp = torch.cuda.ExternalStream(scmp.value, device=dev)
        self.s_out = torch.cuda.ExternalStream(sout.value, device=dev)

    @staticmethod
    def _host(t, shape, name):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a bf16 host tensor")
        if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous {tuple(shape)}")
        if not t.is_pinned():
            raise ValueError(f"{name} must be in pinned (page-locked) memory")
        return ctypes.c_void_p(t.data_ptr())

    def submit(self, hQ, hK, hV, hO):
        """Queue one step: hQ, hK, hV (pinned, the step's inputs) in, O out
        to hO (pinned).  Returns at once; synchronize() waits."""
        _check(_lib.qsa_prefill_pipeline_submit(self._h, self._host(hQ, self.shape_q, "hQ"),
                                                self._host(hK, self.shape_kv, "hK"),
                                                self._host(hV, self.shape_kv, "hV"),
                                                self._host(hO, self.shape_q, "hO")),
               "qsa_prefill_pipeline_submit")

    def synchronize(self):
        _check(_lib.qsa_prefill_pipeline_synchronize(self._h), "qsa_prefill_pipeline_synchronize")

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _lib.qsa_prefill_pipeline_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class QSADecode:
    """The whole decode path for a batch of single-token queries: select
    (per token) then split-K attention.  Summaries of complete blocks are
    persistent state; compress_block() adds one as it completes."""

    def __init__(self, B, Hq, Hkv, d, T_kv_max, topk, device="cuda", summary_dtype=torch.float32):
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, d
        self.T_kv_max, self.topk = T_kv_max, topk
        self.sm_scale = d ** -0.5
        dev = torch.device(device)
        # summaries: fp32, or bf16 (half the bytes the per-token selection reads)
        self.Kc = torch.zeros((B, Hkv, T_kv_max // BLOCK, d), dtype=summary_dtype, device=dev)
        self.idx = torch.empty((B, Hkv, 1, topk), dtype=torch.int32, device=dev)
        self.o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
        n = decode_workspace(B, Hq, Hkv, d, topk)
        self.ws_dec = torch.empty(n, dtype=torch.uint8, device=dev) if n > 0 else None
        self._sel_ws = {}

    def compress(self, K, blk_begin, blk_end, stream=None):
        compress_keys(K, self.Kc, blk_begin, blk_end, stream)

    def __call__(self, q, K, V, L, stream=None):
        q4 = q.view(self.B, 1, self.Hq, self.d)
        key = L
        if key not in self._sel_ws:
            n = score_select_workspace(self.B, self.Hq, self.Hkv, 1, L - 1, 1, self.d, self.topk)
            self._sel_ws[key] = torch.empty(max(1, n), dtype=torch.uint8, device=q.device)
        score_select(q4, self.Kc, self.idx, self.topk, L - 1, 1, self.sm_scale,
                     self._sel_ws[key], stream)
        decode(q, K, V, self.idx, self.o, L, self.sm_scale, self.ws_dec, stream)
        return self.o

    def graph(self, q, K, V, L, parts=("select", "attention")):
        """Capture the step (or some of its parts) for these buffers and this
        cache length as a CUDA graph; ``replay()`` then reruns it on the
        current stream with no host launch work.  The step runs once eagerly
        first (kernel loading, attributes and the selection workspace stay
        out of the capture)."""
        q4 = q.view(self.B, 1, self.Hq, self.d)
        self(q, K, V, L)
        side = torch.cuda.Stream(device=q.device)
        side.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            if "select" in parts:
                score_select(q4, self.Kc, self.idx, self.topk, L - 1, 1, self.sm_scale,
                             self._sel_ws[L], side)
            if "attention" in parts:
                decode(q, K, V, self.idx, self.o, L, self.sm_scale, self.ws_dec, side)
        torch.cuda.current_stream().wait_stream(side)
        return g
