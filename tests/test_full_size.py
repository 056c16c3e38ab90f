"""Parity at the workloads' full sizes, run the way bench.py runs them.

The whole path runs on the GPU at full size (QSAPrefill / QSADecode, the
same objects and launch configuration the benchmark times); the oracle then
recomputes the outputs:
  * selection: every row of every workload -- exact indices where the
    oracle's m-th / (m+1)-th score gap exceeds 1e-3, a valid top-m under the
    oracle's fp64 scores everywhere;
  * attention, over the GPU's own selection: every output element of
    prefill_32k, chunked_1m and every decode sequence; at prefill_128k the
    first 256 tokens (the fewest keys and the largest |O|, where the bf16
    output's own rounding is largest) plus 3840 tokens drawn at random and
    the last token.
Gate: max |err| <= 1e-2 and mean |err| <= 1e-3 over all compared elements;
each test prints the max, the mean and the 99.99th percentile of |err|.
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


def _stats(name, err):
    err = np.asarray(err, dtype=np.float64).ravel()
    q = float(np.quantile(err, 0.9999))
    print(f"FULLSIZE {name}: {err.size} outputs, max|err| {err.max():.3e} mean {err.mean():.3e} "
          f"p99.99 {q:.3e}")


PREFILL = [("prefill_32k", None), ("chunked_1m", None), ("prefill_128k", 4096)]


@pytest.mark.parametrize("name,ntok", PREFILL, ids=[p[0] for p in PREFILL])
def test_prefill_full_size(qsa, name, ntok):
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

    # key summaries: fp32 on the GPU, fp64 in the oracle
    Kc_ref = oracle.compress_keys(Kh)
    rel = np.abs(Kc_gpu - Kc_ref).max() / np.abs(Kc_ref).max()
    assert rel < 1e-5, rel
    # every selection row
    Qbar = oracle.pool_queries(Qh, w.Hkv, w.qblk)
    sel = oracle.select(Qbar, Kc_ref, w.Tq, w.q_pos0, w.qblk, w.topk, w.sm_scale, want_scores=True)
    flat = {"idx": sel["idx"].reshape(-1, w.topk), "gap": sel["gap"].reshape(-1)}
    frac, jac = check_selection(idx.reshape(-1, w.topk), flat, sel["scores"], rows_diag(w), w.topk)
    exact = float(np.mean(np.all(idx.reshape(-1, w.topk) == flat["idx"], axis=-1)))
    print(f"FULLSIZE {name}: {flat['idx'].shape[0]} selection rows, gap-checked {frac:.3f}, "
          f"identical {exact:.3f}, Jaccard {jac:.4f}")
    # attention over the GPU's own selection
    if ntok is None:
        toks = None
        O_gpu = O.float().cpu().numpy().reshape(w.B * w.Tq, w.Hq, w.d)
    else:
        rng = np.random.RandomState(17)
        rest = rng.choice(np.arange(256, w.B * w.Tq - 1), size=ntok - 256, replace=False)
        toks = np.unique(np.concatenate([np.arange(256), rest, [w.B * w.Tq - 1]]))
        O_gpu = O.reshape(w.B * w.Tq, w.Hq, w.d)[torch.from_numpy(toks).to(O.device)].float().cpu().numpy()
    O_ref = oracle.attend(Qh, Kh, Vh, idx, w.q_pos0, w.qblk, w.sm_scale, tokens=toks)
    O_ref = O_ref.reshape(O_gpu.shape)
    _stats(name, np.abs(O_gpu - O_ref))
    check_out(O_gpu, O_ref)


DECODE = [("decode_128k", "fp32"), ("decode_262k", "fp32"), ("decode_128k", "bf16")]


@pytest.mark.parametrize("name,summary", DECODE, ids=[f"{n}-{s}" for n, s in DECODE])
def test_decode_full_size(qsa, name, summary):
    """Every one of the 32 sequences: selection rows and outputs."""
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

    errs, fracs, jacs = [], [], []
    for b in range(w.B):
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
        fracs.append(frac)
        jacs.append(jac)
        O_ref = oracle.attend(qb, Kb, Vb, idx[b:b + 1], w.q_pos0, 1, w.sm_scale)
        errs.append(np.abs(o[b] - O_ref.reshape(w.Hq, w.d)))
        del Kb, Vb
    print(f"FULLSIZE {name} ({summary} summaries): {w.B * w.Hkv} selection rows, gap-checked "
          f"{np.mean(fracs):.3f}, Jaccard {np.mean(jacs):.4f}")
    err = np.stack(errs)
    _stats(f"{name} ({summary} summaries)", err)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
    del x, q, K, V, dec, g
    torch.cuda.empty_cache()
