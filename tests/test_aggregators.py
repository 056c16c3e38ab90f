"""Per-token selection with other ways of combining the group's heads than
the pooled query: the softmax-sum aggregator (each head's softmax over the
complete blocks before the token's diagonal, summed over the heads) and the
max-over-tokens aggregator (for one token per row, the mean).  The pages
have the selector score compressed keys against the queries and leave the
combination open (page "Qwen4 in llama.cpp: Dissecting PR #27742", section
"QSA Is an Address-Selection Problem, Not a New Attention Equation").

The GPU's indices are compared with the oracle's selection rule applied to
the oracle's fp64 scores under the same aggregator, from the same fp32
summaries: exact on rows whose m-th/(m+1)-th score gap exceeds 1e-3, a
valid top-m (to 1e-5) everywhere.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.helpers import check_selection

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_compress_b200 as m
    assert torch.cuda.is_available()
    return m


def _ok(qsa):
    st = qsa.device_status()
    assert st[0] == "QSA_OK", st


CASES = [
    # name, B, Tq, q_pos0, Hq, Hkv, d, topk, plant fraction, plant scale
    ("planted_g8", 4, 1, 64 * 60 + 4, 16, 2, 128, 8, 0.2, 4.0),
    ("tokens_g4_d64", 2, 3, 64 * 150 + 2, 8, 2, 64, 16, 0.1, 3.0),
    ("long_multichunk", 2, 1, 64 * 3000 - 1, 16, 2, 128, 32, 0.02, 4.0),
    # more than 8 x 1024 candidates: chunks too long to keep the softmax-sum
    # logits in shared memory (they are recomputed)
    ("very_long_recompute", 1, 1, 64 * 9000 - 1, 16, 2, 128, 16, 0.002, 4.0),
]


@pytest.mark.parametrize("agg", ["softmax_sum", "max"])
@pytest.mark.parametrize("name,B,Tq,q_pos0,Hq,Hkv,d,topk,frac,scale", CASES, ids=[c[0] for c in CASES])
def test_token_aggregator_parity(qsa, agg, name, B, Tq, q_pos0, Hq, Hkv, d, topk, frac, scale):
    nblk = (q_pos0 + Tq + 63) // 64
    w = synthetic.custom(B=B, Tq=Tq, T_kv=64 * nblk, q_pos0=q_pos0, qblk=1, Hq=Hq, Hkv=Hkv, d=d, topk=topk,
                         seed=211, plant="token", plant_frac=frac, plant_scale=scale)
    x = synthetic.generate(w)
    Kc = torch.from_numpy(oracle.compress_keys(x["K"], 0, nblk).astype(np.float32))   # the summaries both sides use
    idx = torch.full((B, Hkv, Tq, topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_token_agg(x["Q"].to(DEV), Kc.to(DEV), idx, topk, q_pos0, agg, w.sm_scale)
    _ok(qsa)
    s = oracle.block_scores(x["Q"], Kc.double().numpy(), Tq, q_pos0, 1, w.sm_scale, agg)
    sel = oracle.select_scores(s, B, Hkv, Tq, q_pos0, 1, topk)
    NB = s.shape[-1]
    D = [(q_pos0 + i) // 64 for b in range(B) for g in range(Hkv) for i in range(Tq)]
    frac_checked, jac = check_selection(idx.cpu().numpy().reshape(-1, topk), sel, s.reshape(-1, NB), D, topk)
    print(f"{agg} {name}: rows gap-checked {frac_checked:.3f}, Jaccard {jac:.4f}")
    if agg == "softmax_sum" and name == "planted_g8":
        assert frac_checked > 0.5          # the planted blocks give clear gaps here
    if agg == "max":
        # one token per row: the maximum over tokens is the mean, the same kernel
        ref = torch.full_like(idx, -7)
        qsa.score_select_token_agg(x["Q"].to(DEV), Kc.to(DEV), ref, topk, q_pos0, "mean", w.sm_scale)
        assert torch.equal(idx, ref)


def test_token_softmax_sum_ragged(qsa):
    """Per-sequence lengths (one decode token each), softmax-sum aggregator."""
    lens = [64 * 40 + 7, 64 * 300, 130, 64 * 2 + 1, 64 * 77]
    Hq, Hkv, d, topk = 16, 2, 128, 16
    max_blocks = max((L + 63) // 64 for L in lens) + 1
    Kc_all = torch.zeros((len(lens), Hkv, max_blocks, d), dtype=torch.float32)
    qs, refs = [], []
    for b, L in enumerate(lens):
        w = synthetic.custom(B=1, Tq=1, T_kv=64 * max_blocks, q_pos0=L - 1, qblk=1, Hq=Hq, Hkv=Hkv, d=d,
                             topk=topk, seed=221 + b, plant="token", plant_frac=0.2, plant_scale=4.0)
        x = synthetic.generate(w)
        Kc = oracle.compress_keys(x["K"], 0, L // 64).astype(np.float32)
        Kc_all[b, :, :L // 64] = torch.from_numpy(Kc[0, :, :L // 64])
        qs.append(x["Q"])
        s = oracle.block_scores(x["Q"], Kc_all[b:b + 1].double().numpy(), 1, L - 1, 1, w.sm_scale,
                                "softmax_sum")
        refs.append((s, oracle.select_scores(s, 1, Hkv, 1, L - 1, 1, topk), (L - 1) // 64))
    q = torch.cat(qs, 0).to(DEV)
    idx = torch.full((len(lens), Hkv, 1, topk), -7, dtype=torch.int32, device=DEV)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=DEV)
    qsa.score_select_token_agg(q, Kc_all.to(DEV), idx, topk, max(lens) - 1, "softmax_sum", d ** -0.5,
                               seq_lens=seq_lens)
    _ok(qsa)
    idx_h = idx.cpu().numpy()
    for b, (s, sel, D) in enumerate(refs):
        frac_checked, jac = check_selection(idx_h[b].reshape(-1, topk), sel, s.reshape(Hkv, -1), [D] * Hkv, topk)
        print(f"ragged softmax-sum seq {b} (L={lens[b]}): gap-checked {frac_checked:.2f}, Jaccard {jac:.4f}")


def test_token_softmax_sum_full_size(qsa):
    """decode_128k (32 sequences at 131072 tokens, top-64), softmax-sum,
    sampled sequences against the oracle."""
    w = synthetic.CONFIGS["decode_128k"]
    x = synthetic.generate(w, DEV)
    L = w.q_pos0 + 1
    Kc = torch.zeros((w.B, w.Hkv, w.T_kv // 64, w.d), dtype=torch.float32, device=DEV)
    qsa.compress_keys(x["K"], Kc, 0, L // 64)
    idx = torch.full((w.B, w.Hkv, 1, w.topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_token_agg(x["Q"], Kc, idx, w.topk, w.q_pos0, "softmax_sum", w.sm_scale)
    _ok(qsa)
    Kc_h = Kc.cpu().double().numpy()
    Q_h = x["Q"].cpu()
    idx_h = idx.cpu().numpy()
    del x
    torch.cuda.empty_cache()
    D = (L - 1) // 64
    for b in (0, 13, w.B - 1):
        s = oracle.block_scores(Q_h[b:b + 1], Kc_h[b:b + 1], 1, w.q_pos0, 1, w.sm_scale, "softmax_sum")
        sel = oracle.select_scores(s, 1, w.Hkv, 1, w.q_pos0, 1, w.topk)
        frac_checked, jac = check_selection(idx_h[b].reshape(-1, w.topk), sel, s.reshape(w.Hkv, -1),
                                            [D] * w.Hkv, w.topk)
        print(f"decode_128k softmax-sum seq {b}: gap-checked {frac_checked:.2f}, Jaccard {jac:.4f}")


PREFILL_MAX = [
    # name, B, Tq, q_pos0, Hq, Hkv, topk, plant fraction
    ("g4_ragged_tail", 1, 200, 64 * 5, 8, 2, 8, 0.3),
    ("g8_three_tiles", 2, 256, 64 * 300, 16, 2, 16, 0.1),
    ("g8_chunked_rows", 1, 128, 64 * 3000, 16, 2, 32, 0.02),
    # last query block of 32 tokens: its second 32-token half has no valid
    # token and its query tile reaches into the next sequence's rows
    ("g8_ragged_b2", 2, 224, 64 * 40, 16, 2, 16, 0.1),
]


@pytest.mark.parametrize("agg", ["max", "softmax_sum"])
@pytest.mark.parametrize("name,B,Tq,q_pos0,Hq,Hkv,topk,frac", PREFILL_MAX, ids=[c[0] for c in PREFILL_MAX])
def test_prefill_aggregator_parity(qsa, agg, name, B, Tq, q_pos0, Hq, Hkv, topk, frac):
    """Prefill rows under the max-over-tokens and softmax-sum aggregators
    (tensor-core logits over bf16 summaries) against the oracle's
    aggregators on the same bf16 summaries."""
    d = 128
    nblk = (q_pos0 + Tq + 63) // 64
    w = synthetic.custom(B=B, Tq=Tq, T_kv=64 * nblk, q_pos0=q_pos0, qblk=64, Hq=Hq, Hkv=Hkv, d=d, topk=topk,
                         seed=231, plant="partner", plant_frac=frac, plant_scale=1.0)
    x = synthetic.generate(w)
    Kc_ref = oracle.compress_keys(x["K"], 0, nblk, summary="bf16")            # bf16 values, fp64
    Kc = torch.from_numpy(Kc_ref).to(torch.bfloat16).to(DEV)                   # exact
    NR = (Tq + 63) // 64
    idx = torch.full((B, Hkv, NR, topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_prefill_agg(x["Q"].to(DEV), Kc, idx, topk, q_pos0, agg, w.sm_scale)
    _ok(qsa)
    s = oracle.block_scores(x["Q"], Kc_ref, Tq, q_pos0, 64, w.sm_scale, agg)
    sel = oracle.select_scores(s, B, Hkv, Tq, q_pos0, 64, topk)
    D = [(q_pos0 + min((i + 1) * 64, Tq) - 1) // 64 for b in range(B) for g in range(Hkv) for i in range(NR)]
    frac_checked, jac = check_selection(idx.cpu().numpy().reshape(-1, topk), sel, s.reshape(-1, s.shape[-1]), D,
                                        topk)
    print(f"prefill {agg} {name}: rows gap-checked {frac_checked:.3f}, Jaccard {jac:.4f}")


FULL_ROWS = {
    # per workload: sampled selection rows (row r = (b*Hkv + g)*NR + i) --
    # the first rows (fewest candidates), middle and last rows of both groups
    "prefill_32k": lambda NR: [0, 1, 2, 63, 200, 255, 256, 400, 511, NR + 3, NR + 300, 2 * NR - 1],
    "prefill_128k": lambda NR: [0, 1, 2, 5, 700, 1024, 1500, 2047, NR + 3, NR + 1000, NR + 1800, 2 * NR - 1],
}


@pytest.mark.parametrize("wname", ["prefill_32k", "prefill_128k"])
@pytest.mark.parametrize("agg", ["max", "softmax_sum"])
def test_prefill_aggregator_full_size(qsa, agg, wname):
    """The benchmark's workloads (bf16 summaries; 32768 tokens top-16 and
    131072 tokens top-32), sampled rows against the oracle."""
    w = synthetic.CONFIGS[wname]
    x = synthetic.generate(w, DEV)
    nblk = w.T_kv // 64
    Kc = torch.empty((w.B, w.Hkv, nblk, w.d), dtype=torch.bfloat16, device=DEV)
    qsa.compress_keys(x["K"], Kc, 0, (w.q_pos0 + w.Tq) // 64)
    NR = w.Tq // 64
    idx = torch.full((w.B, w.Hkv, NR, w.topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_prefill_agg(x["Q"], Kc, idx, w.topk, w.q_pos0, agg, w.sm_scale)
    _ok(qsa)
    idx_h = idx.cpu().numpy().reshape(-1, w.topk)
    Q_h = x["Q"].cpu()
    Kc_h = Kc.float().cpu().double().numpy()
    del x
    rows = np.array(FULL_ROWS[wname](NR), dtype=np.int32)
    s = oracle.block_scores(Q_h, Kc_h, w.Tq, w.q_pos0, 64, w.sm_scale, agg, rows=rows)
    sel = oracle.select_scores(s, w.B, w.Hkv, w.Tq, w.q_pos0, 64, w.topk, rows=rows)
    D = [(w.q_pos0 + min((r % NR + 1) * 64, w.Tq) - 1) // 64 for r in rows]
    frac_checked, jac = check_selection(idx_h[rows], sel, s, D, w.topk)
    print(f"{wname} {agg}: sampled rows gap-checked {frac_checked:.3f}, Jaccard {jac:.4f}")


@pytest.mark.parametrize("agg", ["max", "softmax_sum"])
def test_aggregators_degenerate_rows(qsa, agg):
    """Rows with no candidate (diagonal block 0 or 1) keep only the forced
    blocks; the rows right after them have one or two candidates."""
    d, Hq, Hkv, topk = 128, 16, 2, 8
    # prefill rows from the first block of the sequence (diagonals 0, 1, 2, 3)
    w = synthetic.custom(B=1, Tq=200, T_kv=256, q_pos0=0, qblk=64, Hq=Hq, Hkv=Hkv, d=d, topk=topk, seed=241)
    x = synthetic.generate(w)
    Kc_ref = oracle.compress_keys(x["K"], 0, 4, summary="bf16")
    idx = torch.full((1, Hkv, 4, topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_prefill_agg(x["Q"].to(DEV), torch.from_numpy(Kc_ref).to(torch.bfloat16).to(DEV), idx, topk, 0,
                                 agg, w.sm_scale)
    _ok(qsa)
    s = oracle.block_scores(x["Q"], Kc_ref, 200, 0, 64, w.sm_scale, agg)
    ref = oracle.select_scores(s, 1, Hkv, 200, 0, 64, topk)["idx"].reshape(idx.shape)
    assert np.array_equal(idx.cpu().numpy(), ref)
    assert idx[0, 0, 0].tolist() == [0] + [-1] * (topk - 1)          # diagonal 0: the sink alone
    assert idx[0, 0, 1].tolist() == [0, 1] + [-1] * (topk - 2)       # diagonal 1: sink and diagonal
    # per-token rows at positions in blocks 0, 1 and 2
    for pos in (3, 70, 130):
        wt = synthetic.custom(B=2, Tq=1, T_kv=256, q_pos0=pos, qblk=1, Hq=Hq, Hkv=Hkv, d=d, topk=topk, seed=242)
        xt = synthetic.generate(wt)
        Kc = oracle.compress_keys(xt["K"], 0, 4).astype(np.float32)
        it = torch.full((2, Hkv, 1, topk), -7, dtype=torch.int32, device=DEV)
        qsa.score_select_token_agg(xt["Q"].to(DEV), torch.from_numpy(Kc).to(DEV), it, topk, pos, agg, wt.sm_scale)
        _ok(qsa)
        st = oracle.block_scores(xt["Q"], Kc.astype(np.float64), 1, pos, 1, wt.sm_scale, agg)
        rt = oracle.select_scores(st, 2, Hkv, 1, pos, 1, topk)["idx"].reshape(it.shape)
        assert np.array_equal(it.cpu().numpy(), rt)
