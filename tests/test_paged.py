"""Ragged batches over paged caches (serving): each sequence has its own
length and its 64-token blocks live in pages named by a block table -- the
"cache-cell IDs" the selector's output is turned into (page "Qwen4 in
llama.cpp: Dissecting PR #27742", section "QSA Is an Address-Selection
Problem, Not a New Attention Equation").

The logical caches come from the seeded generator, one sequence at a time;
the test scatters their blocks into randomly permuted physical pages on the
host.  Each sequence is then checked against the oracle run on its own
logical cache at its own position, with the same acceptance as the
contiguous path (indices exact on clear-gap rows, outputs max |err| <= 1e-2
and mean <= 1e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.helpers import check_out, check_selection

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_compress_b200 as m
    assert torch.cuda.is_available()
    return m


def _status(qsa):
    return qsa.device_status()


def build_paged(lens, Hq, Hkv, d, extra_blocks=2, extra_pages=7, seed=81):
    """Logical per-sequence caches and their paged copy.  Returns a dict with
    per-sequence Q/K/V (host), the page pools, the block table and lengths."""
    B = len(lens)
    max_blocks = max((L + 63) // 64 for L in lens) + extra_blocks
    T = 64 * max_blocks
    seqs = []
    for b, L in enumerate(lens):
        w = synthetic.custom(B=1, Tq=1, T_kv=T, q_pos0=L - 1, qblk=1, Hq=Hq, Hkv=Hkv, d=d, topk=4,
                             seed=seed + b)
        seqs.append(synthetic.generate(w))
    num_pages = B * max_blocks + extra_pages
    rng = np.random.RandomState(seed)
    table = rng.permutation(num_pages)[:B * max_blocks].reshape(B, max_blocks).astype(np.int32)
    K_pages = torch.zeros((num_pages, Hkv, 64, d), dtype=torch.bfloat16)
    V_pages = torch.zeros_like(K_pages)
    for b, x in enumerate(seqs):
        Kb = x["K"][0].view(Hkv, max_blocks, 64, d).permute(1, 0, 2, 3)   # [blocks, Hkv, 64, d]
        Vb = x["V"][0].view(Hkv, max_blocks, 64, d).permute(1, 0, 2, 3)
        idx = torch.from_numpy(table[b].astype(np.int64))
        K_pages[idx] = Kb
        V_pages[idx] = Vb
    q = torch.cat([x["Q"][:, 0] for x in seqs], 0)        # [B, Hq, d]
    return dict(B=B, max_blocks=max_blocks, num_pages=num_pages, seqs=seqs, table=table,
                K_pages=K_pages, V_pages=V_pages, q=q, lens=list(lens))


CASES = [
    ("d128_g8", [64 * 150 - 5, 64 * 300, 64 * 77 + 31, 1000, 64 * 41 + 1], 16, 2, 128, 16),
    ("d64_g4", [64 * 90 + 17, 130, 64 * 200 - 1, 64 * 3], 8, 2, 64, 8),
]


@pytest.mark.parametrize("name,lens,Hq,Hkv,d,topk", CASES, ids=[c[0] for c in CASES])
def test_ragged_paged_decode(qsa, name, lens, Hq, Hkv, d, topk):
    p = build_paged(lens, Hq, Hkv, d)
    B, max_blocks = p["B"], p["max_blocks"]
    sm_scale = d ** -0.5
    K_pages, V_pages = p["K_pages"].to(DEV), p["V_pages"].to(DEV)
    table = torch.from_numpy(p["table"]).to(DEV)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=DEV)
    q = p["q"].to(DEV)
    Kc = torch.full((B, Hkv, max_blocks, d), float("nan"), dtype=torch.float32, device=DEV)
    qsa.compress_keys_paged(K_pages, table, seq_lens, Kc)
    idx = torch.full((B, Hkv, 1, topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_ragged(q.view(B, 1, Hq, d), Kc, seq_lens, idx, topk, max(lens), sm_scale)
    o = torch.full_like(q, float("nan"))
    qsa.decode_paged(q, K_pages, V_pages, table, seq_lens, idx, o, sm_scale)
    st = _status(qsa)
    assert st[0] == "QSA_OK", st
    Kc_h, idx_h, o_h = Kc.cpu().double().numpy(), idx.cpu().numpy(), o.float().cpu().numpy()
    for b, (x, L) in enumerate(zip(p["seqs"], lens)):
        ncomplete = L // 64
        Kc_ref = oracle.compress_keys(x["K"], 0, ncomplete)
        # complete blocks: within the fp32 summation bound; the rest untouched
        ref = Kc_ref[0, :, :ncomplete]
        assert np.abs(Kc_h[b, :, :ncomplete] - ref).max() <= 64 * 2.0 ** -24 * 8 + 1e-12
        assert np.isnan(Kc_h[b, :, ncomplete:]).all()
        Qbar = oracle.pool_queries(x["Q"], Hkv, 1)
        sel = oracle.select(Qbar, Kc_ref, 1, L - 1, 1, topk, sm_scale, rows=np.arange(Hkv),
                            want_scores=True)
        D = (L - 1) // 64
        check_selection(idx_h[b].reshape(Hkv, topk), sel, sel["scores"], [D] * Hkv, topk)
        O_ref = oracle.attend(x["Q"], x["K"][:, :, :L], x["V"][:, :, :L], idx_h[b:b + 1], L - 1, 1,
                              sm_scale)
        mx, mean = check_out(o_h[b], O_ref.reshape(Hq, d))
        print(f"{name} seq {b} (L={L}): o max {mx:.2e} mean {mean:.2e}")


def test_paged_bounds_are_reported(qsa):
    """A page outside the pool and a length past the capacity are caught on
    the device (QSA_ERR_BOUNDS) before any access; the call returns and the
    context stays usable."""
    lens = [64 * 20 + 5, 64 * 30]
    p = build_paged(lens, 8, 2, 64, extra_pages=0)
    B, max_blocks = p["B"], p["max_blocks"]
    K_pages, V_pages = p["K_pages"].to(DEV), p["V_pages"].to(DEV)
    table = torch.from_numpy(p["table"]).to(DEV)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=DEV)
    q = p["q"].to(DEV)
    idx = torch.tensor([[0, 5, 20, -1]] * 2 + [[0, 7, 29, -1]] * 2, dtype=torch.int32,
                       device=DEV).view(B, 2, 1, 4)
    o = torch.empty_like(q)
    _status(qsa)
    bad_table = table.clone()
    bad_table[0, 5] = p["num_pages"] + 3          # a selected block's page is outside the pool
    qsa.decode_paged(q, K_pages, V_pages, bad_table, seq_lens, idx, o)
    assert _status(qsa)[0] == "QSA_ERR_BOUNDS"
    bad_lens = torch.tensor([lens[0], 64 * max_blocks + 1], dtype=torch.int32, device=DEV)
    qsa.decode_paged(q, K_pages, V_pages, table, bad_lens, idx, o)
    assert _status(qsa)[0] == "QSA_ERR_BOUNDS"
    assert torch.equal(o[1].float(), torch.zeros_like(o[1].float()))   # invalid length: zeros
    Kc = torch.zeros((B, 2, max_blocks, 64), dtype=torch.float32, device=DEV)
    qsa.compress_keys_paged(K_pages, bad_table, seq_lens, Kc)
    assert _status(qsa)[0] == "QSA_ERR_BOUNDS"
    assert _status(qsa)[0] == "QSA_OK"


def test_ragged_prefill_position_past_the_plan_is_reported(qsa):
    """A chunk position above the max_pos the selection was planned for
    (device data) is reported as QSA_ERR_BOUNDS -- the row's scores would
    not fit the score table sized for max_pos -- and that sequence is
    treated as starting at 0; the other sequences are selected as usual."""
    B, Tq, Hq, Hkv, d, topk, max_blocks = 2, 128, 8, 2, 64, 6, 64
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    Q = torch.randn((B, Tq, Hq, d), generator=g, device=DEV).to(torch.bfloat16)
    Kc = torch.randn((B, Hkv, max_blocks, d), generator=g, device=DEV) / 8
    idx = torch.full((B, Hkv, 2, topk), -7, dtype=torch.int32, device=DEV)
    good = torch.tensor([64 * 20, 64 * 30], dtype=torch.int32, device=DEV)
    qsa.score_select_ragged_prefill(Q, Kc, good, idx, topk, 64 * 30)
    assert _status(qsa)[0] == "QSA_OK"
    ref = idx.clone()
    past = torch.tensor([64 * 20, 64 * 40], dtype=torch.int32, device=DEV)   # 64 * 40 > max_pos
    idx.fill_(-7)
    qsa.score_select_ragged_prefill(Q, Kc, past, idx, topk, 64 * 30)
    assert _status(qsa)[0] == "QSA_ERR_BOUNDS"
    assert torch.equal(idx[0], ref[0])                     # the valid sequence is untouched by the error
    assert (idx[1, :, :, 0] == 0).all()                    # the invalid one keeps the sink
    assert _status(qsa)[0] == "QSA_OK"


PREFILL_CASES = [
    # name, chunk start per sequence (multiples of 64), Tq, Hq, Hkv, d, topk
    ("d128_g8", [64 * 40, 64 * 100, 0], 192, 16, 2, 128, 8),
    ("d64_g4_ragged_tail", [64 * 7, 64 * 65], 100, 8, 2, 64, 6),
]


@pytest.mark.parametrize("name,qpos,Tq,Hq,Hkv,d,topk", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
def test_ragged_paged_chunked_prefill(qsa, name, qpos, Tq, Hq, Hkv, d, topk):
    """Chunked prefill of several requests at different cache positions over
    paged caches: compress the complete blocks, select per (sequence, query
    block) and attend, each sequence against the oracle on its own logical
    cache."""
    lens = [q + Tq for q in qpos]
    p = build_paged(lens, Hq, Hkv, d, seed=91)
    B, max_blocks = p["B"], p["max_blocks"]
    sm_scale = d ** -0.5
    # the chunk's queries of each sequence (the generator draws Q per sequence)
    Qs = []
    for b, q0 in enumerate(qpos):
        w = synthetic.custom(B=1, Tq=Tq, T_kv=64 * max_blocks, q_pos0=q0, qblk=64, Hq=Hq, Hkv=Hkv, d=d,
                             topk=topk, seed=191 + b)
        Qs.append(synthetic.generate(w)["Q"])
    Q = torch.cat(Qs, 0)
    K_pages, V_pages = p["K_pages"].to(DEV), p["V_pages"].to(DEV)
    table = torch.from_numpy(p["table"]).to(DEV)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=DEV)
    q_pos = torch.tensor(qpos, dtype=torch.int32, device=DEV)
    Kc = torch.zeros((B, Hkv, max_blocks, d), dtype=torch.float32, device=DEV)
    qsa.compress_keys_paged(K_pages, table, seq_lens, Kc)
    NR = (Tq + 63) // 64
    idx = torch.full((B, Hkv, NR, topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_ragged_prefill(Q.to(DEV), Kc, q_pos, idx, topk, max(qpos), sm_scale)
    O = torch.full((B, Tq, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=DEV)
    qsa.sparse_attn_prefill_paged(Q.to(DEV), K_pages, V_pages, table, q_pos, idx, O, sm_scale, lse)
    st = _status(qsa)
    assert st[0] == "QSA_OK", st
    idx_h, O_h, lse_h = idx.cpu().numpy(), O.float().cpu().numpy(), lse.cpu().numpy()
    for b, (x, q0) in enumerate(zip(p["seqs"], qpos)):
        L = q0 + Tq
        Kc_ref = oracle.compress_keys(x["K"], 0, L // 64)
        Qbar = oracle.pool_queries(Qs[b], Hkv, 64)
        sel = oracle.select(Qbar, Kc_ref, Tq, q0, 64, topk, sm_scale, rows=np.arange(Hkv * NR),
                            want_scores=True)
        D = [(q0 + min((i + 1) * 64, Tq) - 1) // 64 for g in range(Hkv) for i in range(NR)]
        check_selection(idx_h[b].reshape(Hkv * NR, topk), sel, sel["scores"], D, topk)
        O_ref, lse_ref = oracle.attend(Qs[b], x["K"][:, :, :L], x["V"][:, :, :L], idx_h[b:b + 1], q0, 64,
                                       sm_scale, want_lse=True)
        mx, mean = check_out(O_h[b], O_ref[0])
        assert np.abs(lse_h[b] - lse_ref[0]).max() <= 1e-3
        print(f"{name} seq {b} (chunk at {q0}): O max {mx:.2e} mean {mean:.2e}")
