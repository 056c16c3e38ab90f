"""fp64 CPU oracle of the QSA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
and its binding) never imports it and never falls back to it.

The arithmetic lives in ``qsa_oracle.c`` (plain fp64 C); this module only
marshals numpy arrays.  bf16 tensors are passed as their raw uint16 bit
patterns.  Sources: the pages "Qwen4 architecture: QSA, GR, PLE" (section
"1. QSA: not looking at every token equally") and "Qwen4 in llama.cpp:
Dissecting PR #27742" (section "QSA Is an Address-Selection Problem, Not a
New Attention Equation").

Parity status of each function is stated in its docstring; every function
here is pinned by ``tests/test_oracle_pins.py``.
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

BLOCK = 64  # key block size fixed by the build's parameterization

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        Dd = ctypes.c_double
        lib.qsa_oracle_threads.restype = I
        lib.qsa_oracle_compress_keys.argtypes = [P, I, I, I, I, I, I, I, P]
        lib.qsa_oracle_compress_keys.restype = None
        lib.qsa_oracle_round_bf16.argtypes = [P, ctypes.c_int64, P]
        lib.qsa_oracle_round_bf16.restype = None
        lib.qsa_oracle_fwht_f32.argtypes = [P, ctypes.c_int64, I]
        lib.qsa_oracle_fwht_f32.restype = None
        lib.qsa_oracle_e4m3.argtypes = [P, ctypes.c_int64, P]
        lib.qsa_oracle_e4m3.restype = None
        lib.qsa_oracle_quantize_rows_fp8.argtypes = [P, ctypes.c_int64, I, P, P]
        lib.qsa_oracle_quantize_rows_fp8.restype = None
        lib.qsa_oracle_pool_queries.argtypes = [P, I, I, I, I, I, I, P]
        lib.qsa_oracle_pool_queries.restype = None
        lib.qsa_oracle_select.argtypes = [P, P, I, I, I, I, I, I, I, I, I, I, Dd,
                                          P, I, P, P, P, P]
        lib.qsa_oracle_select.restype = I
        lib.qsa_oracle_attend.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, I,
                                          Dd, P, I, P, P]
        lib.qsa_oracle_attend.restype = I
        lib.qsa_oracle_block_scores.argtypes = [P, P, I, I, I, I, I, I, I, I, I, Dd, I, P, I, P]
        lib.qsa_oracle_block_scores.restype = I
        lib.qsa_oracle_select_scores.argtypes = [P, I, I, I, I, I, I, I, I, I, P, I, P, P, P]
        lib.qsa_oracle_select_scores.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bits(x):
    """bf16 data as a C-contiguous uint16 array (accepts torch bf16 or uint16)."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("bf16 inputs must be torch.bfloat16 or raw uint16 bits")
    return x


def threads() -> int:
    """Threads the oracle's parallel loops use."""
    return int(_load().qsa_oracle_threads())


def round_bf16(x):
    """Each value rounded to the nearest bf16, ties to even (returned as
    fp64).  Pinned by exact cases and by torch's fp32 -> bf16 conversion."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().qsa_oracle_round_bf16(_ptr(x), x.size, _ptr(y))
    return y


def compress_keys(K, blk_begin=0, blk_end=None, blk=BLOCK, summary="fp32"):
    """Mean-pooled key summaries, fp64.

    K: bf16 [B, H, T, d].  Returns Kc [B, H, T//blk, d]; only blocks in
    [blk_begin, blk_end) are written (others are zero).  summary="bf16" is
    the bf16-summary option: the exact mean rounded to the nearest bf16.
    """
    K = _bits(K)
    B, H, T, d = K.shape
    NB = T // blk
    if blk_end is None:
        blk_end = NB
    assert 0 <= blk_begin <= blk_end <= NB
    Kc = np.zeros((B, H, NB, d), dtype=np.float64)
    _load().qsa_oracle_compress_keys(_ptr(K), B, H, T, d, blk, blk_begin, blk_end, _ptr(Kc))
    if summary == "bf16":
        Kc = round_bf16(Kc)
    elif summary != "fp32":
        raise ValueError(f"summary must be 'fp32' or 'bf16', got {summary!r}")
    return Kc


def pool_queries(Q, Hkv, qblk=BLOCK):
    """Pooled query of each selection row, fp64.  Q: bf16 [B, Tq, Hq, d].
    Returns Qbar [B, Hkv, ceil(Tq/qblk), d]."""
    Q = _bits(Q)
    B, Tq, Hq, d = Q.shape
    assert Hq % Hkv == 0
    NR = -(-Tq // qblk)
    Qbar = np.zeros((B, Hkv, NR, d), dtype=np.float64)
    _load().qsa_oracle_pool_queries(_ptr(Q), B, Tq, Hq, Hkv, d, qblk, _ptr(Qbar))
    return Qbar


def select(Qbar, Kc, Tq, q_pos0, qblk, topk, sm_scale, rows=None, blk=BLOCK,
           want_scores=False):
    """Score + top-k select.  Returns dict with ``idx`` ([nrows, topk] int32,
    or [B, Hkv, NR, topk] when rows is None), ``gap``, ``m`` and optionally
    ``scores`` ([nrows, NB], NaN for non-candidates)."""
    Qbar = np.ascontiguousarray(Qbar, dtype=np.float64)
    Kc = np.ascontiguousarray(Kc, dtype=np.float64)
    B, Hkv, NR, d = Qbar.shape
    NB = Kc.shape[2]
    assert Kc.shape[:2] == (B, Hkv) and Kc.shape[3] == d
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    nrows = B * Hkv * NR if rows is None else len(rows_arr)
    idx = np.empty((nrows, topk), dtype=np.int32)
    gap = np.empty(nrows, dtype=np.float64)
    m = np.empty(nrows, dtype=np.int32)
    scores = np.empty((nrows, NB), dtype=np.float64) if want_scores else None
    rc = _load().qsa_oracle_select(_ptr(Qbar), _ptr(Kc), B, Hkv, NR, NB, d, Tq, q_pos0,
                                   qblk, blk, topk, float(sm_scale), _ptr(rows_arr), nrows,
                                   _ptr(idx), _ptr(gap), _ptr(m), _ptr(scores))
    if rc != 0:
        raise ValueError("oracle select: topk must be >= 2")
    if rows is None:
        idx = idx.reshape(B, Hkv, NR, topk)
        gap = gap.reshape(B, Hkv, NR)
        m = m.reshape(B, Hkv, NR)
    out = {"idx": idx, "gap": gap, "m": m}
    if want_scores:
        out["scores"] = scores
    return out


AGGREGATORS = {"mean": 0, "max": 1, "softmax_sum": 2}


def block_scores(Q, Kc, Tq, q_pos0, qblk, sm_scale, aggregator, rows=None, blk=BLOCK):
    """Per-row block scores under an aggregator of the per-(head, token)
    logits ("mean", "max" over tokens of the head mean, or "softmax_sum" of
    each (head, token)'s softmax over the blocks before the diagonal).
    Q: bf16 [B, Tq, Hq, d]; Kc: [B, Hkv, NB, d].  Returns [nrows, NB] fp64
    (or [B, Hkv, NR, NB] when rows is None), s_j for j < D and NaN elsewhere."""
    Q = _bits(Q)
    Kc = np.ascontiguousarray(Kc, dtype=np.float64)
    B, Tq_, Hq, d = Q.shape
    assert Tq_ == Tq
    _, Hkv, NB, _ = Kc.shape
    NR = -(-Tq // qblk)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    nrows = B * Hkv * NR if rows is None else len(rows_arr)
    out = np.empty((nrows, NB), dtype=np.float64)
    rc = _load().qsa_oracle_block_scores(_ptr(Q), _ptr(Kc), B, Tq, Hq, Hkv, NB, d, q_pos0, qblk, blk,
                                         float(sm_scale), AGGREGATORS[aggregator], _ptr(rows_arr), nrows,
                                         _ptr(out))
    assert rc == 0
    return out.reshape(B, Hkv, NR, NB) if rows is None else out


def select_scores(scores, B, Hkv, Tq, q_pos0, qblk, topk, rows=None, blk=BLOCK):
    """The selection rule on a score table ([nrows, NB], candidates j in
    1..D-1 of each row).  Returns a dict like select()."""
    NR = -(-Tq // qblk)
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    NB = scores.shape[-1]
    scores = scores.reshape(-1, NB)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    nrows = scores.shape[0]
    idx = np.empty((nrows, topk), dtype=np.int32)
    gap = np.empty(nrows, dtype=np.float64)
    m = np.empty(nrows, dtype=np.int32)
    rc = _load().qsa_oracle_select_scores(_ptr(scores), B, Hkv, NR, NB, Tq, q_pos0, qblk, blk, topk,
                                          _ptr(rows_arr), nrows, _ptr(idx), _ptr(gap), _ptr(m))
    if rc != 0:
        raise ValueError("oracle select: topk must be >= 2")
    return {"idx": idx, "gap": gap, "m": m}


def attend(Q, K, V, idx, q_pos0, qblk, sm_scale, tokens=None, blk=BLOCK, want_lse=False):
    """Exact softmax attention over the selected blocks, fp64.

    Q: bf16 [B, Tq, Hq, d]; K, V: bf16 [B, Hkv, T_kv, d];
    idx: int32 [B, Hkv, NR, topk].  Returns O [ntok, Hq, d] for the listed
    flat tokens (b*Tq + t), or [B, Tq, Hq, d] when tokens is None.
    """
    Q, K, V = _bits(Q), _bits(K), _bits(V)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    B, Tq, Hq, d = Q.shape
    _, Hkv, T_kv, _ = K.shape
    NR = -(-Tq // qblk)
    assert idx.shape[:3] == (B, Hkv, NR), (idx.shape, (B, Hkv, NR))
    topk = idx.shape[3]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    ntok = B * Tq if tokens is None else len(tok)
    O = np.empty((ntok, Hq, d), dtype=np.float64)
    lse = np.empty((ntok, Hq), dtype=np.float64) if want_lse else None
    rc = _load().qsa_oracle_attend(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), B, Tq, Hq, Hkv,
                                   T_kv, d, q_pos0, qblk, blk, topk, float(sm_scale),
                                   _ptr(tok), ntok, _ptr(O), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle attend: a selected block lies outside the cache "
                         "or after its query token")
    if tokens is None:
        O = O.reshape(B, Tq, Hq, d)
        if want_lse:
            lse = lse.reshape(B, Tq, Hq)
    return (O, lse) if want_lse else O


def qsa_forward(Q, K, V, Hkv, topk, q_pos0=0, qblk=BLOCK, sm_scale=None, blk=BLOCK,
                tokens=None):
    """The whole path: compress -> pool -> score/select -> attend.

    Keys of the cache (and of the new tokens) sit in K/V [B, Hkv, T_kv, d];
    the Tq query tokens sit at positions q_pos0 .. q_pos0+Tq-1.
    Returns (sel dict, O).
    """
    Qb = _bits(Q)
    d = Qb.shape[3]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    Tq = Qb.shape[1]
    T_kv = _bits(K).shape[2] if not hasattr(K, "shape") else K.shape[2]
    n_complete = (q_pos0 + Tq) // blk
    Kc = compress_keys(K, 0, min(n_complete, T_kv // blk), blk=blk)
    Qbar = pool_queries(Q, Hkv, qblk)
    sel = select(Qbar, Kc, Tq, q_pos0, qblk, topk, sm_scale, blk=blk)
    O = attend(Q, K, V, sel["idx"], q_pos0, qblk, sm_scale, tokens=tokens, blk=blk)
    return sel, O


# ------------------------------------------- one sequence over several GPUs
# The cache of one long sequence split by contiguous block ranges, one per
# rank (the long-context regime of page "Qwen4 in llama.cpp: Dissecting PR
# #27742", section "Why Short-Context Tests Can Lie"): each rank keeps the
# top m of its own candidates by the same order (score descending, block
# ascending), and the union of the ranks' lists holds the row's top m (a
# candidate outside its rank's list has m better ones there).  Attention
# over disjoint key sets combines through their log-sum-exp: with
# L = log sum_r exp(lse_r), O = sum_r exp(lse_r - L) O_r.

def select_shard(Qbar, Kc, Tq, q_pos0, topk, sm_scale, blk_lo, blk_hi, qblk=BLOCK):
    """A rank's candidate lists: for every row, the top m (the row's m, as
    select() sets it) of the candidates j in [blk_lo, blk_hi) with
    1 <= j < D, ordered by (score descending, block ascending).  Returns
    (scores, blocks), each [nrows, 62] (fp64 padded with -inf, int32 padded
    with -1), rows flat (b, g, i) like select(rows=...)."""
    sel = select(Qbar, Kc, Tq, q_pos0, qblk, topk, sm_scale, rows=np.arange(int(np.prod(Qbar.shape[:3]))),
                 want_scores=True)
    scores, m = sel["scores"], sel["m"]
    nrows = len(m)
    NR = Qbar.shape[2]
    out_s = np.full((nrows, 62), -np.inf)
    out_j = np.full((nrows, 62), -1, dtype=np.int32)
    for r in range(nrows):
        i = r % NR
        D = (q_pos0 + min((i + 1) * qblk, Tq) - 1) // BLOCK
        js = np.arange(max(1, blk_lo), min(D - 1, blk_hi - 1) + 1)
        if len(js) == 0 or m[r] == 0:
            continue
        order = sorted(js.tolist(), key=lambda j: (-scores[r, j], j))[:m[r]]
        out_s[r, :len(order)] = scores[r, order]
        out_j[r, :len(order)] = order
    return out_s, out_j


def merge_shard_lists(scores, blocks, Tq, q_pos0, topk, qblk=BLOCK):
    """The rows' selection from all ranks' lists (scores, blocks: [R, nrows,
    L]): the top m of their union by (score descending, block ascending),
    plus blocks 0 and D, ascending, padded with -1 to topk.  Returns idx
    [nrows, topk] int32."""
    R, nrows, _ = blocks.shape
    idx = np.full((nrows, topk), -1, dtype=np.int32)
    NR = -(-Tq // qblk)
    for r in range(nrows):
        i = r % NR
        D = (q_pos0 + min((i + 1) * qblk, Tq) - 1) // BLOCK
        forced = [0] if D == 0 else [0, D]
        m = min(topk - len(forced), max(D - 1, 0))
        cand = [(float(scores[k, r, e]), int(blocks[k, r, e])) for k in range(R)
                for e in range(blocks.shape[2]) if blocks[k, r, e] >= 0]
        chosen = [j for _, j in sorted(cand, key=lambda t: (-t[0], t[1]))[:m]]
        row = sorted(set(forced) | set(chosen))
        idx[r, :len(row)] = row
    return idx


def merge_partials(O_parts, lse_parts):
    """Outputs of attention over disjoint key sets merged by their
    log-sum-exp, fp64: O_parts [R, ..., d], lse_parts [R, ...] (-inf for an
    empty set).  Returns (O, lse)."""
    O_parts = np.asarray(O_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    mx = lse_parts.max(axis=0)
    safe = np.where(np.isfinite(mx), mx, 0.0)
    w = np.exp(lse_parts - safe)                       # exp(-inf) = 0
    tot = w.sum(axis=0)
    O = (w[..., None] * O_parts).sum(axis=0) / np.where(tot > 0, tot, 1.0)[..., None]
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return O, lse


# ------------------------------------------------------- quantized KV option
# Page "Qwen4 in llama.cpp: Dissecting PR #27742", section "Quantized KV
# Exposed a Backend Storage Invariant": K/V stored in a Hadamard-rotated
# basis, attention in the rotated basis, the output returned to the original
# basis (H^2 = I for the normalised transform).  Codes are fp8 e4m3 with one
# fp32 scale per (token, head); the code decisions are fp32 (as the kernels
# take them), the attention fp64.

def fwht_f32(x):
    """Unnormalised Walsh-Hadamard transform of the last axis (n = 64 or
    128), fp32, in the kernels' butterfly order.  Returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32).copy()
    n = x.shape[-1]
    _load().qsa_oracle_fwht_f32(_ptr(x), x.size // n, n)
    return x


def e4m3(x):
    """fp32 values -> fp8 e4m3 codes (uint8): nearest, ties to even,
    saturating to +-448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    c = np.empty(x.shape, dtype=np.uint8)
    _load().qsa_oracle_e4m3(_ptr(x), x.size, _ptr(c))
    return c


def e4m3_value(codes):
    """fp8 e4m3 codes -> their values (fp64), from the format's definition:
    exponent field 0 gives m * 2^-9, otherwise 2^(e - 7) * (1 + m / 8)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e, m = (c >> 3) & 0xF, c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    return sign * mag


def quantize_kv_fp8(X):
    """Rotated fp8 cache: X bf16 [..., n] -> (codes uint8 [..., n], scales
    fp32 [...]) with u = WHT(x) in fp32, s = max|u| / 448, code = e4m3(u / s)."""
    Xb = _bits(X)
    n = Xb.shape[-1]
    rows = Xb.size // n
    codes = np.empty(Xb.shape, dtype=np.uint8)
    scales = np.empty(Xb.shape[:-1], dtype=np.float32)
    _load().qsa_oracle_quantize_rows_fp8(_ptr(Xb), rows, n, _ptr(codes), _ptr(scales))
    return codes, scales


def hadamard(n):
    """Sylvester Hadamard matrix (entries +-1), fp64."""
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def decode_fp8(q, codes_K, scales_K, codes_V, scales_V, idx, L, sm_scale, blk=BLOCK):
    """Decode attention over a rotated fp8 cache, fp64.  q bf16 [B, Hq, n];
    codes uint8 [B, Hkv, T, n]; scales fp32 [B, Hkv, T]; idx int32
    [B, Hkv, 1, topk] (-1 padding); L = cache length (token at L - 1).
    Scores u_q . u_k / n (= q . k), output H o' / n back in the original
    basis.  Returns o [B, Hq, n]."""
    qb = _bits(q)
    qf = _bf16_f64(qb)
    B, Hq, n = qf.shape
    Hkv = codes_K.shape[1]
    G = Hq // Hkv
    H = hadamard(n)
    uq = qf @ H                              # rows: H is symmetric
    o = np.zeros((B, Hq, n))
    for b in range(B):
        for g in range(Hkv):
            keys = []
            for j in np.asarray(idx[b, g]).reshape(-1):
                if j < 0:
                    continue
                keys.extend(range(int(j) * blk, min(int(j) * blk + blk, L)))
            keys = np.array(keys, dtype=np.int64)
            # dequantized rows of the visible keys: code value times row scale
            Kr = e4m3_value(codes_K[b, g, keys]) * np.asarray(scales_K[b, g, keys], dtype=np.float64)[:, None]
            Vr = e4m3_value(codes_V[b, g, keys]) * np.asarray(scales_V[b, g, keys], dtype=np.float64)[:, None]
            for h in range(g * G, (g + 1) * G):
                z = (Kr @ uq[b, h]) / n * sm_scale
                w = np.exp(z - z.max())
                w /= w.sum()
                o[b, h] = H @ (w @ Vr) / n
    return o


def _bf16_f64(bits):
    """uint16 bf16 bit patterns -> fp64 values (exact widening)."""
    u = np.asarray(bits, dtype=np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
