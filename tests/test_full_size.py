"""Parity at the workloads' full sizes, run the way bench.py runs them.

The whole path runs on the GPU at full size (QSAPrefill / QSADecode, the
same objects and launch configuration the benchmark times); the oracle then
recomputes a sample of the outputs one by one: the selection of sampled
rows (exact indices where the k-th / (k+1)-th score gap exceeds 1e-3, a
valid top-m everywhere), and the attention output of sampled tokens over
the GPU's own selection (max |err| <= 1e-2, mean |err| <= 1e-3).  The
samples always include the first and the last rows and tokens, and tokens
inside a partial diagonal block.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.helpers import check_out, check_selection, rows_diag

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_compress_b200 as m
    assert torch.cuda.is_available()
    return m


def _status_ok(qsa):
    st, det = qsa.device_status()
    assert st == "QSA_OK", (st, det)


def _sample(n, k, rng, always=()):
    pick = set(int(a) % n for a in always)
    pick.update(int(x) for x in rng.choice(n, size=min(k, n), replace=False))
    return np.array(sorted(pick), dtype=np.int64)


PREFILL = ["prefill_32k", "prefill_128k", "chunked_1m"]


@pytest.mark.parametrize("name", PREFILL)
def test_prefill_full_size(qsa, name):
    w = synthetic.CONFIGS[name]
    x = synthetic.generate(w, DEV)
    Q, K, V = x["Q"], x["K"], x["V"]
    run = qsa.QSAPrefill(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0, device=DEV)
    run.precompress_cache(K)
    O = run(Q, K, V).clone()
    _status_ok(qsa)
    idx = run.idx.cpu().numpy()
    Kc_gpu = run.Kc.cpu().numpy()
    Qh, Kh, Vh = Q.cpu(), K.cpu(), V.cpu()
    del x, Q, K, V, run
    torch.cuda.empty_cache()

    rng = np.random.RandomState(17)
    NR = w.n_rows
    # key summaries: fp32 on the GPU, fp64 in the oracle
    Kc_ref = oracle.compress_keys(Kh)
    rel = np.abs(Kc_gpu - Kc_ref).max() / np.abs(Kc_ref).max()
    assert rel < 1e-5, rel
    # selection of sampled rows (flat (b, g, i)): first, last, random
    rows = _sample(w.B * w.Hkv * NR, 40, rng, always=(0, NR - 1, NR, -1))
    Qbar = oracle.pool_queries(Qh, w.Hkv, w.qblk)
    sel = oracle.select(Qbar, Kc_ref, w.Tq, w.q_pos0, w.qblk, w.topk, w.sm_scale, rows=rows,
                        want_scores=True)
    D = np.array(rows_diag(w))[rows]
    frac, jac = check_selection(idx.reshape(-1, w.topk)[rows], sel, sel["scores"], D, w.topk)
    # attention of sampled tokens over the GPU's selection
    toks = _sample(w.B * w.Tq, 48, rng, always=(0, 1, 63, 64, w.Tq - 1, w.Tq // 2 + 37))
    O_ref = oracle.attend(Qh, Kh, Vh, idx, w.q_pos0, w.qblk, w.sm_scale, tokens=toks)
    O_gpu = O.reshape(w.B * w.Tq, w.Hq, w.d)[torch.from_numpy(toks).to(O.device)].float().cpu()
    emax, emean = check_out(O_gpu.numpy(), O_ref)
    print(f"{name}: rows gap-checked {frac:.3f}, Jaccard {jac:.4f}; O max {emax:.2e} mean {emean:.2e}")


DECODE = [("decode_128k", "fp32"), ("decode_262k", "fp32"), ("decode_128k", "bf16")]


@pytest.mark.parametrize("name,summary", DECODE, ids=[f"{n}-{s}" for n, s in DECODE])
def test_decode_full_size(qsa, name, summary):
    w = synthetic.CONFIGS[name]
    x = synthetic.generate(w, DEV)
    q = x["Q"].view(w.B, w.Hq, w.d)
    K, V = x["K"], x["V"]
    L = w.q_pos0 + 1
    sdt = torch.bfloat16 if summary == "bf16" else torch.float32
    dec = qsa.QSADecode(w.B, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, device=DEV, summary_dtype=sdt)
    dec.compress(K, 0, L // 64)
    g = dec.graph(q, K, V, L)     # the step as the benchmark replays it
    dec.o.fill_(0)
    dec.idx.fill_(-7)
    g.replay()
    torch.cuda.synchronize()
    _status_ok(qsa)
    idx = dec.idx.cpu().numpy()               # [B, Hkv, 1, topk]
    o = dec.o.float().cpu().numpy()           # [B, Hq, d]
    Kc_gpu = dec.Kc.cpu().double().numpy()

    rng = np.random.RandomState(23)
    seqs = _sample(w.B, 3, rng, always=(0, w.B - 1))
    for b in seqs:
        Kb, Vb = K[b:b + 1].cpu(), V[b:b + 1].cpu()
        qb = x["Q"][b:b + 1].cpu()           # [1, 1, Hq, d]
        Kc_ref = oracle.compress_keys(Kb, 0, L // 64, summary=summary)
        # fp32: the fp32 summation error; bf16: at most one bf16 rounding step
        # (the exact and the fp32 mean can round to neighbours at a boundary)
        tol = 1e-5 if summary == "fp32" else 2.0 ** -7
        rel = np.abs(Kc_gpu[b:b + 1, :, :L // 64] - Kc_ref[:, :, :L // 64]).max() / np.abs(Kc_ref).max()
        assert rel < tol, rel
        Qbar = oracle.pool_queries(qb, w.Hkv, 1)
        sel = oracle.select(Qbar, Kc_ref, 1, w.q_pos0, 1, w.topk, w.sm_scale,
                            rows=np.arange(w.Hkv), want_scores=True)
        D = [(L - 1) // 64] * w.Hkv
        frac, jac = check_selection(idx[b].reshape(-1, w.topk), sel, sel["scores"], D, w.topk)
        O_ref = oracle.attend(qb, Kb, Vb, idx[b:b + 1], w.q_pos0, 1, w.sm_scale)
        emax, emean = check_out(o[b], O_ref.reshape(w.Hq, w.d))
        print(f"{name} ({summary} summaries) seq {b}: rows gap-checked {frac:.3f}, Jaccard {jac:.4f}; "
              f"o max {emax:.2e} mean {emean:.2e}")
    del x, q, K, V, dec, g
    torch.cuda.empty_cache()
