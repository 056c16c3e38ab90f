"""GPU parity: each CUDA step, called through the C ABI, against the fp64
oracle on the same seeded inputs.

Acceptance (the build's tolerance for bf16 I/O with fp32 accumulation):
  * block indices: exactly the oracle's wherever the oracle's m-th/(m+1)-th
    score gap exceeds 1e-3; in every row, the GPU's chosen set must be a
    valid top-m under the oracle's fp64 scores up to 1e-5 (fp32 scoring
    error is ~1e-7), plus the structural rules (ascending, unique, sink and
    diagonal kept, -1 padding);
  * outputs: max |err| <= 1e-2 and mean |err| <= 1e-3 against fp64;
  * key summaries: within the recursive-summation bound
    64 * 2^-24 * mean(|K|) of the exact mean;
  * lse: |err| <= 1e-3.
Cases span several tiles, ragged tails, cache offsets, multi-chunk
selection rows and both head dims / group sizes.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests.helpers import check_out, check_selection, jaccard, rows_diag

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


def gpu_kc(qsa, K):
    B, H, T, d = K.shape
    Kc = torch.zeros((B, H, T // 64, d), dtype=torch.float32, device=DEV)
    qsa.compress_keys(K, Kc)
    return Kc


# ------------------------------------------------------------------ tests
def test_bounded_wait_reports_timeout(qsa):
    """A wait on an mbarrier nothing completes runs out, records
    QSA_ERR_TIMEOUT, and leaves the context usable."""
    qsa.device_status()
    qsa.selftest_wait_timeout(1_000_000)
    st, det = qsa.device_status()
    assert st == "QSA_ERR_TIMEOUT" and det == 99
    assert qsa.device_status()[0] == "QSA_OK"
    torch.ones(4, device=DEV).sum().item()


def test_fma_pipe_exp2_against_cuda_exp2(qsa):
    """The polynomial 2^x the prefill softmax runs on the FMA pipe, against
    CUDA's exp2 on the same device: relative error <= 1e-4 on [-125, 8]
    (the bf16 rounding of P that follows is 2^-9); tiny at and below -126,
    where the result is subnormal."""
    import ctypes
    g = torch.Generator(device=DEV).manual_seed(5)
    x = torch.cat([torch.rand(1 << 20, generator=g, device=DEV) * 133.0 - 125.0,
                   torch.linspace(-1.0, 1.0, 4097, device=DEV),
                   torch.tensor([0.0, 8.0, -0.5, 0.5, -125.0], device=DEV)])
    y = torch.empty_like(x)
    rc = qsa.lib().qsa_selftest_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                     x.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= 1e-4, rel
    low = torch.tensor([-126.0, -127.0, -500.0, float("-inf")], device=DEV)
    yl = torch.empty_like(low)
    qsa.lib().qsa_selftest_exp2(ctypes.c_void_p(low.data_ptr()), ctypes.c_void_p(yl.data_ptr()), 4,
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert (yl >= 0).all() and (yl <= 2.0 ** -125).all()


def test_fma_pipe_softmax_weight_exp2_against_cuda_exp2(qsa):
    """The degree-5 polynomial 2^x the softmax-sum selection passes run on
    the FMA pipe for a share of their weights, against CUDA's exp2 on the
    same device: relative error <= 4e-7 on [-125, 0] (ex2.approx itself is
    within 2^-22 = 2.4e-7 of 2^x); tiny at and below -126."""
    import ctypes
    g = torch.Generator(device=DEV).manual_seed(6)
    x = torch.cat([-torch.rand(1 << 20, generator=g, device=DEV) * 125.0,
                   torch.linspace(-2.0, 0.0, 8193, device=DEV),
                   torch.tensor([0.0, -0.5, -1.5, -125.0], device=DEV)])
    y = torch.empty_like(x)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = qsa.lib().qsa_selftest_exp2_weight(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                            x.numel(), stream)
    assert rc == 0
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= 4e-7, rel
    low = torch.tensor([-126.0, -127.0, -500.0, float("-inf")], device=DEV)
    yl = torch.empty_like(low)
    qsa.lib().qsa_selftest_exp2_weight(ctypes.c_void_p(low.data_ptr()), ctypes.c_void_p(yl.data_ptr()), 4, stream)
    assert (yl >= 0).all() and (yl <= 2.0 ** -125).all()


@pytest.mark.parametrize("d", [64, 128])
def test_compress_parity_and_reproducibility(qsa, d):
    w = synthetic.custom(B=2, Tq=64, T_kv=1280, Hq=8, Hkv=2, d=d, seed=21)
    x = synthetic.generate(w)
    K = x["K"].to(DEV)
    Kc = gpu_kc(qsa, K)
    _status_ok(qsa)
    ref = oracle.compress_keys(x["K"])
    bound = 64 * 2.0 ** -24 * np.abs(x["K"].double().numpy()).reshape(2, 2, 20, 64, d).mean(axis=3)
    err = np.abs(Kc.cpu().double().numpy() - ref)
    assert (err <= bound + 1e-30).all(), err.max()
    # incremental (one block as it completes) == whole pass, bit for bit
    Kc2 = torch.full_like(Kc, float("nan"))
    for j in range(20):
        qsa.compress_keys(K, Kc2, j, j + 1)
    assert torch.equal(Kc, Kc2)
    # a sub-range leaves the other blocks untouched
    Kc3 = torch.full_like(Kc, 7.0)
    qsa.compress_keys(K, Kc3, 5, 9)
    assert torch.equal(Kc3[:, :, 5:9], Kc[:, :, 5:9]) and (Kc3[:, :, :5] == 7).all()


@pytest.mark.parametrize("d", [64, 128])
def test_compress_bf16_summaries(qsa, d):
    """bf16-summary option: the GPU's fp32 mean rounded to the nearest bf16.
    Bit-identical to torch's rounding of the GPU's own fp32 summaries (same
    reduction order), and against the oracle (the exact mean rounded) equal
    wherever the exact mean is not within the fp32 summation bound of a
    rounding boundary; elsewhere a valid rounding of a value within the
    bound."""
    w = synthetic.custom(B=2, Tq=64, T_kv=1280, Hq=8, Hkv=2, d=d, seed=22)
    x = synthetic.generate(w)
    K = x["K"].to(DEV)
    Kc32 = gpu_kc(qsa, K)
    Kb = torch.zeros(Kc32.shape, dtype=torch.bfloat16, device=DEV)
    qsa.compress_keys(K, Kb)
    _status_ok(qsa)
    assert torch.equal(Kb, Kc32.to(torch.bfloat16))
    exact = oracle.compress_keys(x["K"])
    ref = oracle.compress_keys(x["K"], summary="bf16")
    got = Kb.cpu().double().numpy()
    bound = 64 * 2.0 ** -24 * np.abs(x["K"].double().numpy()).reshape(2, 2, 20, 64, d).mean(axis=3)
    spacing = np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 2.0 ** -126))) - 7)
    differ = got != ref
    assert (np.abs(got - exact) <= spacing / 2 + bound)[differ].all()
    assert differ.mean() < 1e-3, differ.mean()
    # incremental == whole pass, bit for bit
    Kb2 = torch.full_like(Kb, float("nan"))
    for j in range(20):
        qsa.compress_keys(K, Kb2, j, j + 1)
    assert torch.equal(Kb, Kb2)


SELECT_CASES = [
    # name, custom kwargs
    ("tiny_1k", None),
    ("prefill_offset_d128", dict(B=1, Tq=320, T_kv=1344, q_pos0=1024, Hq=16, Hkv=2, d=128,
                                 topk=8, plant="partner", plant_frac=0.2)),
    ("prefill_ragged_d64", dict(B=2, Tq=200, T_kv=256, q_pos0=0, Hq=8, Hkv=2, d=64, topk=3)),
    ("decode_multichunk", dict(B=4, Tq=1, T_kv=64 * 700, q_pos0=64 * 700 - 1, qblk=1, Hq=16,
                               Hkv=2, d=128, topk=16)),
    ("decode_many_chunks", dict(B=1, Tq=1, T_kv=64 * 5000, q_pos0=64 * 5000 - 30, qblk=1,
                                Hq=8, Hkv=2, d=64, topk=64)),
    # per-token rows inside a prefill chunk (qblk = 1, Tq > 1): ragged diagonals
    ("token_rows_prefill", dict(B=2, Tq=96, T_kv=640, q_pos0=544, qblk=1, Hq=8, Hkv=2, d=64,
                                topk=6)),
    # top-2 leaves only the forced blocks; top-3 chooses one over several chunks
    ("decode_top2", dict(B=3, Tq=1, T_kv=64 * 900, q_pos0=64 * 900 - 7, qblk=1, Hq=16, Hkv=2,
                         d=128, topk=2)),
    ("decode_top3", dict(B=3, Tq=1, T_kv=64 * 900, q_pos0=64 * 900 - 7, qblk=1, Hq=16, Hkv=2,
                         d=128, topk=3)),
]


@pytest.mark.parametrize("name,kw", SELECT_CASES, ids=[c[0] for c in SELECT_CASES])
def test_score_select_parity(qsa, name, kw):
    w = synthetic.CONFIGS["tiny_prefill_1k"] if kw is None else synthetic.custom(seed=31, **kw)
    x = synthetic.generate(w)
    Q, K = x["Q"].to(DEV), x["K"].to(DEV)
    Kc = gpu_kc(qsa, K)
    idx = torch.full((w.B, w.Hkv, w.n_rows, w.topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select(Q, Kc, idx, w.topk, w.q_pos0, w.qblk, w.sm_scale)
    _status_ok(qsa)
    Kc_ref = oracle.compress_keys(x["K"])
    Qbar = oracle.pool_queries(x["Q"], w.Hkv, w.qblk)
    sel = oracle.select(Qbar, Kc_ref, w.Tq, w.q_pos0, w.qblk, w.topk, w.sm_scale, rows=np.arange(w.B * w.Hkv * w.n_rows), want_scores=True)
    frac, jac = check_selection(idx.cpu().numpy().reshape(-1, w.topk), sel, sel["scores"],
                                rows_diag(w), w.topk)
    print(f"{name}: rows gap-checked {frac:.3f}, mean Jaccard {jac:.4f}")


BF16_SELECT_CASES = ["tiny_1k", "prefill_offset_d128", "decode_multichunk", "decode_many_chunks",
                     "token_rows_prefill"]


@pytest.mark.parametrize("name", BF16_SELECT_CASES)
def test_score_select_bf16_summaries(qsa, name):
    """Selection over bf16 summaries, against the oracle scoring its own
    bf16-rounded summaries (the same gap rule and top-m validity)."""
    kw = dict(SELECT_CASES)[name]
    w = synthetic.CONFIGS["tiny_prefill_1k"] if kw is None else synthetic.custom(seed=32, **kw)
    x = synthetic.generate(w)
    Q, K = x["Q"].to(DEV), x["K"].to(DEV)
    Kb = torch.zeros((w.B, w.Hkv, w.T_kv // 64, w.d), dtype=torch.bfloat16, device=DEV)
    qsa.compress_keys(K, Kb)
    idx = torch.full((w.B, w.Hkv, w.n_rows, w.topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select(Q, Kb, idx, w.topk, w.q_pos0, w.qblk, w.sm_scale)
    _status_ok(qsa)
    Kc_ref = oracle.compress_keys(x["K"], summary="bf16")
    Qbar = oracle.pool_queries(x["Q"], w.Hkv, w.qblk)
    sel = oracle.select(Qbar, Kc_ref, w.Tq, w.q_pos0, w.qblk, w.topk, w.sm_scale,
                        rows=np.arange(w.B * w.Hkv * w.n_rows), want_scores=True)
    frac, jac = check_selection(idx.cpu().numpy().reshape(-1, w.topk), sel, sel["scores"],
                                rows_diag(w), w.topk)
    print(f"{name} (bf16 summaries): rows gap-checked {frac:.3f}, mean Jaccard {jac:.4f}")


def test_score_select_token_rows_past_the_cluster_limit(qsa):
    """Per-token rows with more than 8 x 8192 candidates leave the one-launch
    cluster path for the chunked path with a workspace; both must select the
    same blocks as the oracle.  Random summaries stand in for compressed keys
    (only the scoring and selection are under test)."""
    nb = 66000
    w = synthetic.custom(B=1, Tq=1, T_kv=64 * nb, q_pos0=64 * nb - 1, qblk=1, Hq=8, Hkv=2,
                         d=64, topk=24, seed=33)
    assert qsa.score_select_workspace(w.B, w.Hq, w.Hkv, 1, w.q_pos0, 1, w.d, w.topk) > 0
    assert qsa.score_select_workspace(w.B, w.Hq, w.Hkv, 1, 64 * 5000, 1, w.d, w.topk) == 0
    gen = torch.Generator().manual_seed(w.seed)
    Q = torch.randn((w.B, 1, w.Hq, w.d), generator=gen).to(torch.bfloat16)
    Kc = torch.randn((w.B, w.Hkv, nb, w.d), generator=gen) * 0.2
    idx = torch.full((w.B, w.Hkv, 1, w.topk), -7, dtype=torch.int32, device=DEV)
    qsa.score_select(Q.to(DEV), Kc.to(DEV), idx, w.topk, w.q_pos0, 1, w.sm_scale)
    _status_ok(qsa)
    Qbar = oracle.pool_queries(Q, w.Hkv, 1)
    sel = oracle.select(Qbar, Kc.double(), 1, w.q_pos0, 1, w.topk, w.sm_scale,
                        rows=np.arange(w.B * w.Hkv), want_scores=True)
    frac, jac = check_selection(idx.cpu().numpy().reshape(-1, w.topk), sel, sel["scores"],
                                rows_diag(w), w.topk)
    print(f"66000 candidates: rows gap-checked {frac:.3f}, mean Jaccard {jac:.4f}")


@pytest.mark.parametrize("Hq,d", [(16, 128), (8, 128), (16, 64), (8, 64)])
def test_prefill_single_key_row_returns_its_value(qsa, Hq, d):
    """Token 0 of a fresh sequence sees only key 0: softmax weight 1, so
    its output is V[0] of its group bit for bit, whatever the score's sign
    (a row max taken over anything but the visible keys breaks this)."""
    torch.manual_seed(Hq + d)
    B, T, Hkv = 1, 256, 2
    G = Hq // Hkv
    Q = torch.randn(B, T, Hq, d, device=DEV).to(torch.bfloat16)
    K = (torch.randn(B, Hkv, T, d, device=DEV) * 2).to(torch.bfloat16)
    V = (torch.randn(B, Hkv, T, d, device=DEV) * 3).to(torch.bfloat16)
    run = qsa.QSAPrefill(B, T, Hq, Hkv, d, T, 2, 0, device=DEV)
    O = run(Q, K, V)
    _status_ok(qsa)
    assert torch.equal(O[0, 0], V[0, :, 0].repeat_interleave(G, 0))


PREFILL_CASES = [
    ("tiny_1k", None),
    ("d128_g8_offset", dict(B=1, Tq=192, T_kv=704, q_pos0=512, Hq=16, Hkv=2, d=128, topk=5)),
    ("d128_g8_ragged_b2", dict(B=2, Tq=150, T_kv=448, q_pos0=256, Hq=16, Hkv=2, d=128, topk=4)),
    ("d64_g8", dict(B=1, Tq=256, T_kv=256, q_pos0=0, Hq=16, Hkv=2, d=64, topk=3)),
    ("d128_g4_long", dict(B=1, Tq=128, T_kv=4224, q_pos0=4096, Hq=8, Hkv=2, d=128, topk=40)),
]


@pytest.mark.parametrize("name,kw", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
def test_prefill_attention_parity(qsa, name, kw):
    """The attention kernel on the oracle's own selection."""
    w = synthetic.CONFIGS["tiny_prefill_1k"] if kw is None else synthetic.custom(seed=41, **kw)
    x = synthetic.generate(w)
    Kc_ref = oracle.compress_keys(x["K"])
    Qbar = oracle.pool_queries(x["Q"], w.Hkv, 64)
    sel = oracle.select(Qbar, Kc_ref, w.Tq, w.q_pos0, 64, w.topk, w.sm_scale)
    O_ref, lse_ref = oracle.attend(x["Q"], x["K"], x["V"], sel["idx"], w.q_pos0, 64, w.sm_scale,
                                   want_lse=True)
    Q, K, V = (x[k].to(DEV) for k in ("Q", "K", "V"))
    idx = torch.from_numpy(sel["idx"]).to(DEV)
    O = torch.full_like(Q, float("nan"))
    lse = torch.empty((w.B, w.Tq, w.Hq), dtype=torch.float32, device=DEV)
    qsa.sparse_attn_prefill(Q, K, V, idx, O, w.q_pos0, w.sm_scale, lse)
    _status_ok(qsa)
    mx, mean = check_out(O.float().cpu().numpy(), O_ref)
    assert np.abs(lse.cpu().double().numpy() - lse_ref).max() <= 1e-3
    print(f"{name}: O max|err| {mx:.3g} mean {mean:.3g}")


DECODE_CASES = [
    ("d128_g8", dict(B=4, L=1000, T_kv=1024, Hq=16, Hkv=2, d=128, topk=8)),
    ("d64_g4_odd_topk", dict(B=3, L=777, T_kv=832, Hq=8, Hkv=2, d=64, topk=5)),
    ("d128_g8_k64", dict(B=2, L=64 * 40, T_kv=64 * 40, Hq=16, Hkv=2, d=128, topk=64)),
    ("d128_g4_long", dict(B=2, L=64 * 300 + 17, T_kv=64 * 301, Hq=8, Hkv=2, d=128, topk=32)),
]


@pytest.mark.parametrize("name,kw", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_parity(qsa, name, kw):
    L = kw["L"]
    w = synthetic.custom(B=kw["B"], Tq=1, T_kv=kw["T_kv"], q_pos0=L - 1, qblk=1, Hq=kw["Hq"],
                         Hkv=kw["Hkv"], d=kw["d"], topk=kw["topk"], seed=51)
    x = synthetic.generate(w)
    Kh, Vh = x["K"][:, :, :L], x["V"][:, :, :L]
    sel, O_ref = oracle.qsa_forward(x["Q"], Kh, Vh, w.Hkv, w.topk, q_pos0=L - 1, qblk=1)
    q = x["Q"].to(DEV).view(w.B, w.Hq, w.d)
    K, V = x["K"].to(DEV), x["V"].to(DEV)
    idx = torch.from_numpy(sel["idx"]).to(DEV)
    o = torch.full_like(q, float("nan"))
    for _ in range(2):   # the device-side merge tickets must reset between calls
        qsa.decode(q, K, V, idx, o, L, w.sm_scale)
        _status_ok(qsa)
        mx, mean = check_out(o.float().cpu().numpy(), O_ref[:, 0])
    print(f"{name}: o max|err| {mx:.3g} mean {mean:.3g}")


def test_end_to_end_tiny(qsa):
    """The whole path on the tiny workload: every selection row valid (and
    equal to the oracle's where the gap is clear), every output element
    against the oracle's attention over the GPU's own selection."""
    w = synthetic.CONFIGS["tiny_prefill_1k"]
    x = synthetic.generate(w)
    run = qsa.QSAPrefill(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, device=DEV)
    O = run(*(x[k].to(DEV) for k in ("Q", "K", "V")))
    _status_ok(qsa)
    idx = run.idx.cpu().numpy()
    rows = np.arange(w.B * w.Hkv * w.n_rows)
    sel = oracle.select(oracle.pool_queries(x["Q"], w.Hkv, w.qblk), oracle.compress_keys(x["K"]), w.Tq, 0,
                        w.qblk, w.topk, w.sm_scale, rows=rows, want_scores=True)
    check_selection(idx.reshape(-1, w.topk), sel, sel["scores"], rows_diag(w), w.topk)
    O_ref = oracle.attend(x["Q"], x["K"], x["V"], idx, 0, w.qblk, w.sm_scale)
    check_out(O.float().cpu().numpy(), O_ref)
    planted_hit = np.mean([j in idx[b, g, i] for (b, g, j, i) in x["planted"]])
    assert planted_hit > 0.8


def test_bad_block_index_sets_bounds_status(qsa):
    """An index past the row's diagonal is rejected by the kernel (never
    loaded) and reported; the call returns normally."""
    w = synthetic.custom(B=1, Tq=128, T_kv=128, Hq=8, Hkv=2, d=64, topk=3, seed=61)
    x = synthetic.generate(w)
    Q, K, V = (x[k].to(DEV) for k in ("Q", "K", "V"))
    idx = torch.tensor([[[[0, -1, -1], [0, 1, 5]]]] * 1, dtype=torch.int32).repeat(1, 2, 1, 1).to(DEV)
    O = torch.empty_like(Q)
    qsa.sparse_attn_prefill(Q, K, V, idx.contiguous(), O, 0)
    st, det = qsa.device_status()
    assert st == "QSA_ERR_BOUNDS"
    assert qsa.device_status()[0] == "QSA_OK"


def test_prefill_host_pipeline_matches_direct_calls(qsa):
    """The host pipeline (uploads, compute and downloads of neighbouring
    steps on three streams, two device buffer sets) returns for every step
    exactly what a direct call on device tensors returns."""
    w = synthetic.custom(B=1, Tq=320, T_kv=1344, q_pos0=1024, Hq=16, Hkv=2, d=128, topk=8, seed=71)
    inputs = []
    for s in range(3):
        x = synthetic.generate(synthetic.Workload(**{**w.__dict__, "seed": 71 + s}))
        inputs.append({k: x[k].pin_memory() for k in ("Q", "K", "V")})
    ref = []
    for x in inputs:
        run = qsa.QSAPrefill(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0, device=DEV)
        K = x["K"].to(DEV)
        run.precompress_cache(K)
        ref.append(run(x["Q"].to(DEV), K, x["V"].to(DEV)).cpu())
    pipe = qsa.PrefillHostPipeline(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0, device=DEV)
    order = [0, 1, 2, 0, 1, 2]
    outs = [torch.empty_like(ref[s]).pin_memory() for s in order]
    for k, s in enumerate(order):
        x = inputs[s]
        pipe.submit(x["Q"], x["K"], x["V"], outs[k])
    pipe.synchronize()
    _status_ok(qsa)
    for k, s in enumerate(order):
        assert torch.equal(outs[k], ref[s]), f"step {k}"
