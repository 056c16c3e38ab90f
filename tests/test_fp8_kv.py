"""Quantized-KV option for decode: the cache in a Walsh-Hadamard-rotated
basis as fp8 e4m3 codes with a per-row scale, attention in that basis, the
output rotated back (page "Qwen4 in llama.cpp: Dissecting PR #27742",
section "Quantized KV Exposed a Backend Storage Invariant").

The codes and scales are integer-like decisions taken in fp32 on both sides,
so they must match the oracle bit for bit; the attention is compared with
the oracle's fp64 attention over its own codes (max |err| <= 1e-2, mean
<= 1e-3).  The difference from attention over the unquantized cache is the
quantization itself and is only reported.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.helpers import check_out

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_long_compress_b200 as m
    assert torch.cuda.is_available()
    return m


def test_quantize_kv_fp8_matches_oracle_bit_for_bit(qsa):
    w = synthetic.custom(B=2, Tq=1, T_kv=64 * 40, q_pos0=64 * 40 - 1, qblk=1, Hq=16, Hkv=2, d=128, seed=141)
    x = synthetic.generate(w)
    for X in (x["K"], x["V"]):
        codes, scales = qsa.quantize_kv_fp8(X.to(DEV))
        st = qsa.device_status()
        assert st[0] == "QSA_OK", st
        ref_c, ref_s = oracle.quantize_kv_fp8(X)
        assert np.array_equal(codes.cpu().numpy(), ref_c)
        assert np.array_equal(scales.cpu().numpy(), ref_s)
    # an all-zero row quantizes to zero codes and scale
    z = torch.zeros((3, 128), dtype=torch.bfloat16, device=DEV)
    c, s = qsa.quantize_kv_fp8(z)
    assert (c == 0).all() and (s == 0).all()


CASES = [
    ("g8", dict(B=4, T=64 * 300, L=64 * 300 - 9, Hq=16, Hkv=2, topk=16)),
    ("g4_short", dict(B=3, T=64 * 60, L=64 * 41 + 5, Hq=8, Hkv=2, topk=8)),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_decode_fp8_parity(qsa, name, kw):
    L = kw["L"]
    w = synthetic.custom(B=kw["B"], Tq=1, T_kv=kw["T"], q_pos0=L - 1, qblk=1, Hq=kw["Hq"], Hkv=kw["Hkv"],
                         d=128, topk=kw["topk"], seed=151)
    x = synthetic.generate(w)
    sel, O_bf16 = oracle.qsa_forward(x["Q"], x["K"][:, :, :L], x["V"][:, :, :L], w.Hkv, w.topk, q_pos0=L - 1,
                                     qblk=1)
    idx = torch.from_numpy(sel["idx"]).to(DEV)                # [B, Hkv, 1, topk]
    q = x["Q"].to(DEV).view(w.B, w.Hq, 128)
    kc, ks = qsa.quantize_kv_fp8(x["K"].to(DEV))
    vc, vs = qsa.quantize_kv_fp8(x["V"].to(DEV))
    o = torch.full_like(q, float("nan"))
    for _ in range(2):
        qsa.decode_fp8(q, kc, ks, vc, vs, idx, o, L, w.sm_scale)
        st = qsa.device_status()
        assert st[0] == "QSA_OK", st
    ck, sk = oracle.quantize_kv_fp8(x["K"])
    cv, sv = oracle.quantize_kv_fp8(x["V"])
    ref = oracle.decode_fp8(x["Q"].view(w.B, w.Hq, 128), ck, sk, cv, sv, sel["idx"], L, w.sm_scale)
    mx, mean = check_out(o.float().cpu().numpy(), ref)
    qerr = np.abs(ref - O_bf16[:, 0]).max()
    print(f"{name}: o max {mx:.2e} mean {mean:.2e}; quantization vs bf16 cache: max {qerr:.2e}")


@pytest.mark.parametrize("Hq", [16, 8], ids=["g8", "g4"])
def test_decode_fp8_paged_parity(qsa, Hq):
    """A ragged batch over paged rotated fp8 caches: the pages' rows are
    quantized like any rows, each sequence is checked against the oracle's
    fp8 decode on its own logical cache; a page outside the pool is caught
    on the device."""
    from tests.test_paged import build_paged
    lens = [64 * 150 - 5, 64 * 300, 64 * 77 + 31, 1000, 64 * 41 + 1]
    Hkv, d, topk = 2, 128, 16
    p = build_paged(lens, Hq, Hkv, d, seed=171)
    B, max_blocks = p["B"], p["max_blocks"]
    sm = d ** -0.5
    table = torch.from_numpy(p["table"]).to(DEV)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=DEV)
    q = p["q"].to(DEV)
    kc, ks = qsa.quantize_kv_fp8(p["K_pages"].to(DEV))
    vc, vs = qsa.quantize_kv_fp8(p["V_pages"].to(DEV))
    # selection on the unrotated keys' summaries, as the cache write path keeps them
    Kc = torch.zeros((B, Hkv, max_blocks, d), dtype=torch.float32, device=DEV)
    qsa.compress_keys_paged(p["K_pages"].to(DEV), table, seq_lens, Kc)
    idx = torch.full((B, Hkv, 1, topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select_ragged(q.view(B, 1, Hq, d), Kc, seq_lens, idx, topk, max(lens), sm)
    o = torch.full_like(q, float("nan"))
    qsa.decode_fp8_paged(q, kc, ks, vc, vs, table, seq_lens, idx, o, sm)
    st = qsa.device_status()
    assert st[0] == "QSA_OK", st
    idx_h, o_h = idx.cpu().numpy(), o.float().cpu().numpy()
    for b, (x, L) in enumerate(zip(p["seqs"], lens)):
        ck, sk = oracle.quantize_kv_fp8(x["K"])
        cv, sv = oracle.quantize_kv_fp8(x["V"])
        ref = oracle.decode_fp8(x["Q"].view(1, Hq, d), ck, sk, cv, sv, idx_h[b:b + 1], L, sm)
        mx, mean = check_out(o_h[b], ref[0])
        print(f"paged fp8 seq {b} (L={L}): o max {mx:.2e} mean {mean:.2e}")
    bad = table.clone()
    bad[0, int(idx_h[0, 0, 0, 1])] = p["num_pages"] + 3      # a selected block's page is outside the pool
    qsa.decode_fp8_paged(q, kc, ks, vc, vs, bad, seq_lens, idx, o, sm)
    assert qsa.device_status()[0] == "QSA_ERR_BOUNDS"
    assert qsa.device_status()[0] == "QSA_OK"


def test_decode_fp8_full_size(qsa):
    """decode_128k over the rotated fp8 cache, in the benchmark's launch
    configuration (32 sequences at 131072 tokens, top-64, bf16 summaries of
    the unrotated keys): every sequence's codes and scales bit for bit, and
    every output against the oracle's fp8 decode with the GPU's indices."""
    w = synthetic.CONFIGS["decode_128k"]
    x = synthetic.generate(w, DEV)
    L = w.q_pos0 + 1
    q = x["Q"].view(w.B, w.Hq, w.d)
    dec = qsa.QSADecode(w.B, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, device=DEV, summary_dtype=torch.bfloat16)
    dec.compress(x["K"], 0, L // 64)
    qsa.score_select(q.view(w.B, 1, w.Hq, w.d), dec.Kc, dec.idx, w.topk, L - 1, 1, dec.sm_scale)
    kc, ks = qsa.quantize_kv_fp8(x["K"])
    vc, vs = qsa.quantize_kv_fp8(x["V"])
    o = torch.full_like(q, float("nan"))
    qsa.decode_fp8(q, kc, ks, vc, vs, dec.idx, o, L, w.sm_scale)
    st = qsa.device_status()
    assert st[0] == "QSA_OK", st
    idx_h, o_h = dec.idx.cpu().numpy(), o.float().cpu().numpy()
    errs = []
    for b in range(w.B):
        # the oracle quantizes this sequence's rows itself (codes are a
        # per-row function of the row)
        ck, sk = oracle.quantize_kv_fp8(x["K"][b:b + 1].cpu())
        cv, sv = oracle.quantize_kv_fp8(x["V"][b:b + 1].cpu())
        # the codes and scales of the whole sequence, bit for bit
        assert np.array_equal(kc[b:b + 1].cpu().numpy(), ck) and np.array_equal(ks[b:b + 1].cpu().numpy(), sk)
        assert np.array_equal(vc[b:b + 1].cpu().numpy(), cv) and np.array_equal(vs[b:b + 1].cpu().numpy(), sv)
        ref = oracle.decode_fp8(q[b:b + 1].cpu(), ck, sk, cv, sv, idx_h[b:b + 1], L, w.sm_scale)
        errs.append(np.abs(o_h[b] - ref[0]))
    err = np.stack(errs)
    print(f"FULLSIZE decode_128k (rotated fp8 cache): {err.size} outputs, max|err| {err.max():.3e} "
          f"mean {err.mean():.3e} p99.99 {np.quantile(err, 0.9999):.3e}")
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())


@pytest.mark.parametrize("L", [1, 2, 65, 130])
def test_decode_fp8_short_caches(qsa, L):
    """Caches of one token, of a partial first block, and of a few blocks:
    the diagonal block's causal limit and the sink alone.  With one visible
    key the output is that key's value row, of magnitude 1 for N(0, 1)
    values, where the bf16 output's own rounding is already about 1e-3 on
    average; the values are scaled by 1/4 (exact in bf16) so that the
    standard tolerance measures the kernel, as it does for averaged rows."""
    w = synthetic.custom(B=2, Tq=1, T_kv=256, q_pos0=L - 1, qblk=1, Hq=16, Hkv=2, d=128, topk=4, seed=251)
    x = synthetic.generate(w)
    x["V"] = x["V"] * 0.25
    D = (L - 1) // 64
    idx_np = np.full((2, 2, 1, 4), -1, dtype=np.int32)
    for b in range(2):
        for g in range(2):
            blocks = sorted(set([0, D]))
            idx_np[b, g, 0, :len(blocks)] = blocks
    idx = torch.from_numpy(idx_np).to(DEV)
    q = x["Q"].to(DEV).view(2, 16, 128)
    kc, ks = qsa.quantize_kv_fp8(x["K"].to(DEV))
    vc, vs = qsa.quantize_kv_fp8(x["V"].to(DEV))
    o = torch.full_like(q, float("nan"))
    qsa.decode_fp8(q, kc, ks, vc, vs, idx, o, L, w.sm_scale)
    st = qsa.device_status()
    assert st[0] == "QSA_OK", st
    ck, sk = oracle.quantize_kv_fp8(x["K"])
    cv, sv = oracle.quantize_kv_fp8(x["V"])
    ref = oracle.decode_fp8(x["Q"].view(2, 16, 128), ck, sk, cv, sv, idx_np, L, w.sm_scale)
    check_out(o.float().cpu().numpy(), ref)
