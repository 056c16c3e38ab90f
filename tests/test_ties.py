"""Exact score ties in the selection: block 0 and the diagonal are kept and
ties go to the lower block index.  With exactly equal scores the gap rule
exempts a row, so these cases compare the indices with the oracle's
exactly, on inputs whose ties both sides reproduce bit for bit: zero
queries (every score 0) and summaries repeated with a short period (equal
rows give equal dot products in any fixed arithmetic)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_compress_b200 as m
    assert torch.cuda.is_available()
    return m


def _tied(B, Tq, Hq, Hkv, d, nblk, period, zero_q, seed):
    g = torch.Generator().manual_seed(seed)
    Q = torch.zeros((B, Tq, Hq, d)) if zero_q else torch.randn((B, Tq, Hq, d), generator=g)
    Q = Q.to(torch.bfloat16)
    base = torch.randn((B, Hkv, period, d), generator=g)
    reps = -(-nblk // period)
    Kc = base.repeat(1, 1, reps, 1)[:, :, :nblk].contiguous()
    return Q, Kc.float()


CASES = [
    # name, B, Tq, q_pos0, qblk, Hq, Hkv, d, topk, period, zero queries
    ("token_zero_q", 3, 1, 64 * 900 + 5, 1, 16, 2, 128, 64, 7, True),
    ("token_period7", 3, 1, 64 * 900 + 5, 1, 16, 2, 128, 64, 7, False),
    ("token_multichunk_period3", 2, 1, 64 * 5000 - 1, 1, 16, 2, 128, 32, 3, False),
    ("prefill_zero_q", 1, 256, 64 * 300, 64, 8, 2, 64, 16, 5, True),
    ("prefill_period5", 1, 256, 64 * 3000, 64, 16, 2, 128, 32, 5, False),
]


@pytest.mark.parametrize("name,B,Tq,q_pos0,qblk,Hq,Hkv,d,topk,period,zq", CASES, ids=[c[0] for c in CASES])
def test_selection_ties_exact(qsa, name, B, Tq, q_pos0, qblk, Hq, Hkv, d, topk, period, zq):
    nblk = (q_pos0 + Tq + 63) // 64 + 1
    Q, Kc = _tied(B, Tq, Hq, Hkv, d, nblk, period, zq, seed=301)
    NR = -(-Tq // qblk)
    idx = torch.full((B, Hkv, NR, topk), -7, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(16, qsa.score_select_workspace(B, Hq, Hkv, Tq, q_pos0, qblk, d, topk)),
                     dtype=torch.uint8, device=DEV)
    qsa.score_select(Q.to(DEV), Kc.to(DEV), idx, topk, q_pos0, qblk, d ** -0.5, ws)
    st = qsa.device_status()
    assert st[0] == "QSA_OK", st
    Qbar = oracle.pool_queries(Q, Hkv, qblk)
    sel = oracle.select(Qbar, Kc.double().numpy(), Tq, q_pos0, qblk, topk, d ** -0.5)
    assert np.array_equal(idx.cpu().numpy(), sel["idx"])
    if zq:
        # every score is 0: the lowest blocks win
        row = idx[0, 0, 0].cpu().numpy()
        D = (q_pos0 + min(qblk, Tq) - 1) // 64
        m = min(topk - 2, D - 1)
        assert row[:m + 2].tolist() == list(range(m + 1)) + [D]


def test_selection_ties_exact_bf16_and_softmax(qsa):
    """The same ties through the bf16-summary selection and the per-token
    softmax-sum aggregator."""
    B, Tq, q_pos0, Hq, Hkv, d, topk = 2, 1, 64 * 700 + 9, 16, 2, 128, 32
    nblk = (q_pos0 + Tq + 63) // 64 + 1
    Q, Kc = _tied(B, Tq, Hq, Hkv, d, nblk, 4, False, seed=302)
    Kb = Kc.to(torch.bfloat16)
    idx = torch.full((B, Hkv, 1, topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select(Q.to(DEV), Kb.to(DEV), idx, topk, q_pos0, 1, d ** -0.5)
    assert qsa.device_status()[0] == "QSA_OK"
    Qbar = oracle.pool_queries(Q, Hkv, 1)
    sel = oracle.select(Qbar, Kb.double().numpy(), Tq, q_pos0, 1, topk, d ** -0.5)
    assert np.array_equal(idx.cpu().numpy(), sel["idx"])
    idx2 = torch.full_like(idx, -7)
    qsa.score_select_token_agg(Q.to(DEV), Kc.to(DEV), idx2, topk, q_pos0, "softmax_sum", d ** -0.5)
    assert qsa.device_status()[0] == "QSA_OK"
    s = oracle.block_scores(Q, Kc.double().numpy(), Tq, q_pos0, 1, d ** -0.5, "softmax_sum")
    ref = oracle.select_scores(s, B, Hkv, Tq, q_pos0, 1, topk)["idx"].reshape(idx.shape)
    # the softmax-sum is a sum of exponentials: equal logits give equal
    # shares on both sides, so the ties are exact here too
    assert np.array_equal(idx2.cpu().numpy(), ref)
