"""Pins of the fp64 oracle to facts other than itself: closed forms,
invariants, brute force on tiny inputs, and library routines (torch SDPA in
fp64) in the regimes where QSA reduces to plain attention.

The regime pins follow the page "Qwen4 in llama.cpp: Dissecting PR #27742",
section "QSA Is an Address-Selection Problem, Not a New Attention Equation"
(below the budget nothing can be dropped, so sparse equals dense; above it,
compare set overlap), section "The PR's Numerical Evidence Is Layered
Correctly" (a CPU semantic oracle; QSA equals dense below the sparse
threshold), and section "Quantized KV Exposed a Backend Storage Invariant"
(Q' = HQ, K' = HK with H orthonormal preserves Q^T K).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic

BLK = 64


def bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def f64(x_bf16):
    return x_bf16.to(torch.float64).numpy()


def rand_grid(shape, gen, lo=-4.0, hi=4.0, step=0.125):
    """Random values on a coarse grid: exactly representable in bf16, and
    closed under the affine maps the invariance pins apply."""
    n = int(round((hi - lo) / step))
    ints = torch.randint(0, n + 1, shape, generator=gen)
    return bf16(lo + step * ints.to(torch.float32))


# ----------------------------------------------------------------- compress
def test_compress_closed_form_ramp():
    B, H, T, d = 2, 2, 256, 16
    t = torch.arange(T).view(1, 1, T, 1) % BLK
    c = torch.arange(d).view(1, 1, 1, d)
    h = torch.arange(H).view(1, H, 1, 1)
    K = bf16((t + c + 3 * h).expand(B, H, T, d).clone())
    Kc = oracle.compress_keys(K)
    # mean of r = 0..63 is 31.5
    expect = 31.5 + np.arange(d)[None, None, None, :] + 3 * np.arange(H)[None, :, None, None]
    assert np.array_equal(Kc, np.broadcast_to(expect, Kc.shape))


def test_compress_shift_and_block_range():
    g = torch.Generator().manual_seed(1)
    K = rand_grid((1, 2, 512, 32), g)
    Kc = oracle.compress_keys(K, 2, 6)
    Kc_shift = oracle.compress_keys(bf16(K.float() + 1.0), 2, 6)
    assert np.allclose(Kc_shift[:, :, 2:6], Kc[:, :, 2:6] + 1.0, atol=0, rtol=1e-15)
    assert np.all(Kc[:, :, :2] == 0) and np.all(Kc[:, :, 6:] == 0)
    # a constant block compresses to that constant
    Kconst = bf16(torch.full((1, 1, 128, 8), 0.375))
    assert np.all(oracle.compress_keys(Kconst) == 0.375)


def test_compress_page_candidate_count():
    """Page "Qwen4 in llama.cpp", section "Why Short-Context Tests Can Lie":
    262144 positions at compression ratio 4 give 65536 compressed blocks."""
    import json, os
    facts = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))
    f = facts["candidate_count"]
    K = bf16(torch.ones((1, 1, f["n_kv"], 1)))
    Kc = oracle.compress_keys(K, blk=f["ratio"])
    assert Kc.shape[2] == f["blocks"]


def test_round_bf16_exact_cases():
    """The bf16-summary option rounds to the nearest bf16, ties to even:
    values worked out by hand on the 8-significant-bit grid."""
    u = 2.0 ** -7                      # spacing of bf16 in [1, 2)
    cases = [
        (1.0, 1.0),
        (1.0 + u / 2, 1.0),            # tie: the even neighbour is 1
        (1.0 + 3 * u / 2, 1.0 + 2 * u),  # tie: the even neighbour is 1 + 2u
        (1.0 + u / 2 + 2.0 ** -30, 1.0 + u),   # just above the tie: up
        (-(1.0 + 3 * u / 2), -(1.0 + 2 * u)),  # symmetric in sign
        (2.0 - u / 4, 2.0),            # rounds up into the next binade
        (255.5, 256.0),                # 255.5 is a tie at spacing 1: even is 256
        (0.1, 0.10009765625),          # 0.1 = 1.6 * 2^-4 -> 205/128 * 2^-4
        (2.0 ** -130, 2.0 ** -130),    # subnormal, on the grid of 2^-133
        (1.5 * 2.0 ** -133, 2.0 ** -132),  # subnormal tie: even multiple
        (0.0, 0.0),
    ]
    x = np.array([c[0] for c in cases])
    assert np.array_equal(oracle.round_bf16(x), np.array([c[1] for c in cases]))


def test_round_bf16_matches_torch_fp32_conversion():
    """On fp32 inputs, rounding to bf16 is what torch's fp32 -> bf16
    conversion does (round to nearest even): an independent library check."""
    g = torch.Generator().manual_seed(5)
    x32 = torch.randn(20000, generator=g) * torch.exp2(torch.randint(-20, 20, (20000,), generator=g).float())
    # include exact ties: values in [1, 2) of either sign whose 16 dropped
    # bits are 0x8000 (halfway between two bf16 neighbours)
    mant = torch.randint(0, 128, (2000,), generator=g, dtype=torch.int32) << 16
    sign = torch.randint(0, 2, (2000,), generator=g, dtype=torch.int32) << 31
    ties = sign | 0x3F800000 | mant | 0x8000
    x32 = torch.cat([x32, ties.view(torch.float32)])
    assert torch.isfinite(x32).all()
    ref = x32.to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_bf16(x32.to(torch.float64).numpy()), ref)


def test_compress_bf16_option_is_the_rounded_mean():
    g = torch.Generator().manual_seed(6)
    K = bf16(torch.randn((1, 2, 256, 16), generator=g))
    Kc = oracle.compress_keys(K)
    Kb = oracle.compress_keys(K, summary="bf16")
    assert np.array_equal(Kb, oracle.round_bf16(Kc))
    # every value is on the bf16 grid and within half a bf16 spacing
    assert np.array_equal(Kb, f64(bf16(torch.from_numpy(Kb).float())))
    assert np.all(np.abs(Kb - Kc) <= np.abs(Kc) * 2.0 ** -8 + 1e-300)


# --------------------------------------------------------------------- pool
def test_pool_closed_form_with_tail():
    B, Tq, Hq, Hkv, d = 1, 100, 8, 2, 4      # rows: 64 tokens, then a 36-token tail
    t = torch.arange(Tq).view(1, Tq, 1, 1).float()
    h = torch.arange(Hq).view(1, 1, Hq, 1).float()
    c = torch.arange(d).view(1, 1, 1, d).float()
    Q = bf16((t + 10 * h + c).expand(B, Tq, Hq, d).clone())
    Qbar = oracle.pool_queries(Q, Hkv, 64)
    G = Hq // Hkv
    for g in range(Hkv):
        hmean = 10 * (g * G + (G - 1) / 2)
        assert np.allclose(Qbar[0, g, 0], 31.5 + hmean + np.arange(d), rtol=0, atol=1e-12)
        assert np.allclose(Qbar[0, g, 1], (64 + 99) / 2 + hmean + np.arange(d), rtol=0, atol=1e-12)


def test_pool_identity_and_head_permutation():
    g = torch.Generator().manual_seed(2)
    Q = rand_grid((2, 5, 2, 8), g)
    # one head per group, one token per row: pooling is the identity
    Qbar = oracle.pool_queries(Q, 2, 1)
    assert np.array_equal(Qbar.transpose(0, 2, 1, 3), f64(Q))
    Q8 = rand_grid((1, 128, 8, 16), g)
    perm = torch.tensor([2, 0, 3, 1, 7, 5, 4, 6])      # within each group of 4
    a = oracle.pool_queries(Q8, 2, 64)
    b = oracle.pool_queries(Q8[:, :, perm], 2, 64)
    assert np.allclose(a, b, rtol=0, atol=1e-14)


# -------------------------------------------------------------------- score
def _rand_case(seed, Tq=256, T_kv=None, Hq=8, Hkv=2, d=32, topk=4, q_pos0=None, qblk=64):
    w = synthetic.custom(Tq=Tq, T_kv=T_kv, Hq=Hq, Hkv=Hkv, d=d, topk=topk,
                         q_pos0=q_pos0, qblk=qblk, seed=seed)
    return w, synthetic.generate(w)


def test_score_equals_mean_of_per_token_logits():
    """Pooled-query score == mean over (head, token) of each token's logit
    against the block summary (computed here without any pooling)."""
    w, x = _rand_case(3, Tq=192, T_kv=448, q_pos0=256)
    Kc = oracle.compress_keys(x["K"])
    Qbar = oracle.pool_queries(x["Q"], w.Hkv, 64)
    out = oracle.select(Qbar, Kc, w.Tq, w.q_pos0, 64, w.topk, w.sm_scale, want_scores=True)
    S = out["scores"].reshape(w.B, w.Hkv, w.n_rows, -1)
    q = f64(x["Q"])
    G = w.Hq // w.Hkv
    Kbf = f64(x["K"])
    for g in range(w.Hkv):
        for i in range(w.n_rows):
            D = (w.q_pos0 + min((i + 1) * 64, w.Tq) - 1) // 64
            toks = q[0, i * 64:(i + 1) * 64, g * G:(g + 1) * G, :].reshape(-1, w.d)
            for j in range(1, D):
                kc = Kbf[0, g, j * 64:(j + 1) * 64].sum(axis=0) / 64.0
                logits = toks @ kc * w.sm_scale
                assert abs(S[0, g, i, j] - logits.mean()) < 1e-12
            assert np.all(np.isnan(S[0, g, i, D:])) and np.isnan(S[0, g, i, 0])


def test_score_rotation_and_shift_invariance():
    """Q' = HQ, K' = HK with H orthonormal preserves every score; adding one
    vector c to every key shifts a row's scores by a constant, so neither
    changes the selection."""
    w, x = _rand_case(4, Tq=256, T_kv=1024, q_pos0=768, d=32, topk=6)
    Kc = oracle.compress_keys(x["K"])
    Qbar = oracle.pool_queries(x["Q"], w.Hkv, 64)
    base = oracle.select(Qbar, Kc, w.Tq, w.q_pos0, 64, w.topk, w.sm_scale, want_scores=True)
    H, _ = np.linalg.qr(np.random.default_rng(0).standard_normal((w.d, w.d)))
    rot = oracle.select(Qbar @ H.T, Kc @ H.T, w.Tq, w.q_pos0, 64, w.topk, w.sm_scale,
                        want_scores=True)
    m = ~np.isnan(base["scores"])
    assert np.allclose(rot["scores"][m], base["scores"][m], rtol=0, atol=1e-12)
    ok = base["gap"].reshape(-1) > 1e-9
    assert np.array_equal(rot["idx"].reshape(-1, w.topk)[ok], base["idx"].reshape(-1, w.topk)[ok])
    c = np.random.default_rng(1).standard_normal(w.d)
    sh = oracle.select(Qbar, Kc + c, w.Tq, w.q_pos0, 64, w.topk, w.sm_scale, want_scores=True)
    delta = (sh["scores"] - base["scores"]).reshape(w.B, w.Hkv, w.n_rows, -1)
    for g in range(w.Hkv):
        for i in range(w.n_rows):
            row = delta[0, g, i][~np.isnan(delta[0, g, i])]
            assert np.allclose(row, w.sm_scale * Qbar[0, g, i] @ c, rtol=0, atol=1e-12)
    assert np.array_equal(sh["idx"].reshape(-1, w.topk)[ok], base["idx"].reshape(-1, w.topk)[ok])


# ------------------------------------------------------------------- select
def _check_selection(idx_row, scores_row, D, topk):
    """Brute-force validity of one selection row under (score desc, index asc)."""
    sel = [j for j in idx_row if j >= 0]
    assert sel == sorted(set(sel)), "ascending and duplicate-free"
    assert all(0 <= j <= D for j in sel)
    assert 0 in sel and (D == 0 or D in sel), "sink and diagonal always kept"
    assert len(idx_row) == topk
    cand = list(range(1, D))
    chosen = [j for j in sel if 1 <= j < D]
    m = min(topk - (2 if D > 0 else 1), len(cand))
    assert len(chosen) == m
    key = lambda j: (scores_row[j], -j)
    unchosen = [j for j in cand if j not in chosen]
    if chosen and unchosen:
        assert min(key(j) for j in chosen) > max(key(j) for j in unchosen)
    return chosen


def test_select_brute_force_with_ties():
    rng = np.random.default_rng(5)
    for trial in range(30):
        d = 4
        NB = 24
        Kc = rng.integers(-2, 3, size=(1, 1, NB, d)).astype(np.float64)   # many ties
        Qbar = rng.integers(-2, 3, size=(1, 1, 1, d)).astype(np.float64)
        topk = int(rng.integers(2, 10))
        D = int(rng.integers(0, NB))
        q_pos0 = D * 64 + int(rng.integers(0, 64))
        out = oracle.select(Qbar, Kc, 1, q_pos0, 1, topk, 1.0, want_scores=True)
        s = out["scores"][0]
        chosen = _check_selection(list(out["idx"][0, 0, 0]), s, D, topk)
        # brute force over all subsets of the right size
        cand = list(range(1, D))
        m = len(chosen)
        if m == 0 or m == len(cand):
            assert out["gap"][0, 0, 0] == math.inf
            continue
        srt = sorted((s[j] for j in cand), reverse=True)
        assert out["gap"][0, 0, 0] == pytest.approx(srt[m - 1] - srt[m], abs=1e-15)
        if len(cand) <= 14:
            best = None
            for sub in itertools.combinations(cand, m):
                k = sorted(((s[j], -j) for j in sub), reverse=True)
                if best is None or k > best[0]:
                    best = (k, sub)
            assert sorted(best[1]) == chosen


def test_select_special_cases():
    d = 8
    Kc = np.zeros((1, 1, 40, d))
    Qbar = np.zeros((1, 1, 1, d))
    run = lambda q_pos0, topk: oracle.select(Qbar, Kc, 1, q_pos0, 1, topk, 1.0)["idx"][0, 0, 0]
    assert list(run(10, 4)) == [0, -1, -1, -1]                  # D = 0
    assert list(run(64, 4)) == [0, 1, -1, -1]                   # D = 1: no candidates
    assert list(run(64 * 5 + 3, 8)) == [0, 1, 2, 3, 4, 5, -1, -1]  # k >= D+1 keeps all
    # all scores tie: the lowest indices win
    assert list(run(64 * 30, 5)) == [0, 1, 2, 3, 30]
    with pytest.raises(ValueError):
        oracle.select(Qbar, Kc, 1, 100, 1, 1, 1.0)


def test_select_planted_tiny_config_statistic():
    w = synthetic.CONFIGS["tiny_prefill_1k"]
    x = synthetic.generate(w)
    sel, _ = oracle.qsa_forward(x["Q"], x["K"], x["V"], w.Hkv, w.topk, tokens=[0])
    hit = sum(1 for (b, g, j, i) in x["planted"] if j in sel["idx"][b, g, i])
    assert hit >= 0.8 * len(x["planted"])


# ------------------------------------------------------------------ attend
def _sdpa_f64(Q, K, V, mask, scale):
    """torch SDPA in fp64 on [B, Tq, Hq, d] / [B, Hkv, T, d] with GQA expansion."""
    B, Tq, Hq, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    q = Q.to(torch.float64).permute(0, 2, 1, 3)
    k = K.to(torch.float64).repeat_interleave(G, dim=1)
    v = V.to(torch.float64).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def test_attend_dense_equivalence_below_budget():
    """k >= number of causal blocks: nothing can be dropped, QSA equals dense
    causal attention (page: bit identical below the sparse budget).  Against
    torch SDPA in fp64, and bit-identical to itself with a larger k."""
    w, x = _rand_case(6, Tq=300, T_kv=300, Hq=8, Hkv=2, d=32, topk=5)
    sel, O = oracle.qsa_forward(x["Q"], x["K"], x["V"], w.Hkv, 5, q_pos0=0)
    causal = torch.ones(300, 300, dtype=torch.bool).tril()
    ref = _sdpa_f64(x["Q"], x["K"], x["V"], causal, w.sm_scale)
    assert np.abs(O - ref).max() < 1e-12
    _, O9 = oracle.qsa_forward(x["Q"], x["K"], x["V"], w.Hkv, 9, q_pos0=0)
    assert np.array_equal(O, O9)


def test_attend_masked_brute_force_and_decode():
    """Any selection: equals SDPA with the dense T x T mask built from the
    selected blocks (prefill with a cache offset, and per-token decode)."""
    for (Tq, T_kv, q_pos0, qblk, topk, seed) in [(192, 704, 512, 64, 4, 8),
                                                 (3, 900, 897, 1, 5, 9)]:
        w, x = _rand_case(seed, Tq=Tq, T_kv=T_kv, q_pos0=q_pos0, qblk=qblk, topk=topk)
        sel, O = oracle.qsa_forward(x["Q"], x["K"], x["V"], w.Hkv, topk, q_pos0=q_pos0,
                                    qblk=qblk)
        G = w.Hq // w.Hkv
        mask = torch.zeros(w.B, w.Hq, Tq, T_kv, dtype=torch.bool)
        for b in range(w.B):
            for h in range(w.Hq):
                for t in range(Tq):
                    p = q_pos0 + t
                    for j in sel["idx"][b, h // G, t // qblk]:
                        if j >= 0:
                            mask[b, h, t, j * 64:min((j + 1) * 64, p + 1)] = True
        ref = _sdpa_f64(x["Q"], x["K"], x["V"], mask, w.sm_scale)
        assert np.abs(O - ref).max() < 1e-12
        if qblk == 1:
            # decode with every block kept == last rows of dense causal attention
            _, Ofull = oracle.qsa_forward(x["Q"], x["K"], x["V"], w.Hkv, T_kv // 64 + 1,
                                          q_pos0=q_pos0, qblk=1)
            causal = torch.zeros(Tq, T_kv, dtype=torch.bool)
            for t in range(Tq):
                causal[t, :q_pos0 + t + 1] = True
            ref = _sdpa_f64(x["Q"], x["K"], x["V"], causal, w.sm_scale)
            assert np.abs(Ofull - ref).max() < 1e-12


def test_attend_affine_uniform_and_permutation():
    g = torch.Generator().manual_seed(10)
    B, Tq, Hq, Hkv, d, T_kv, topk = 1, 128, 8, 2, 16, 512, 3
    Q = rand_grid((B, Tq, Hq, d), g)
    K = rand_grid((B, Hkv, T_kv, d), g)
    V = rand_grid((B, Hkv, T_kv, d), g)
    idx = np.full((B, Hkv, 2, topk), -1, dtype=np.int32)
    idx[0, :, 0] = [0, 3, 6]
    idx[0, :, 1] = [0, 2, 7]
    q_pos0 = 384
    O = oracle.attend(Q, K, V, idx, q_pos0, 64, 0.25)
    O2 = oracle.attend(Q, K, bf16(2.0 * V.float() + 1.0), idx, q_pos0, 64, 0.25)
    assert np.allclose(O2, 2.0 * O + 1.0, rtol=0, atol=1e-12)
    # zero queries: uniform weights -> mean of the visible values; lse = log(n)
    Z = bf16(torch.zeros_like(Q.float()))
    Oz, lse = oracle.attend(Z, K, V, idx, q_pos0, 64, 0.25, want_lse=True)
    Vf = f64(V)
    for t in [0, 5, 63, 64, 100, 127]:
        p = q_pos0 + t
        blocks = idx[0, 0, t // 64]
        rows = [u for j in blocks for u in range(j * 64, (j + 1) * 64) if u <= p]
        assert np.allclose(Oz[0, t, 0], Vf[0, 0, rows].mean(axis=0), rtol=0, atol=1e-12)
        assert lse[0, t, 0] == pytest.approx(math.log(len(rows)), abs=1e-12)
    # permuting heads within a group permutes the output the same way
    perm = torch.tensor([1, 3, 0, 2, 6, 4, 7, 5])
    Op = oracle.attend(Q[:, :, perm], K, V, idx, q_pos0, 64, 0.25)
    assert np.array_equal(Op, O[:, :, perm.numpy()])
    # an index after the token's position is an error
    bad = idx.copy()
    bad[0, 0, 0, 2] = 7
    with pytest.raises(ValueError):
        oracle.attend(Q, K, V, bad, q_pos0, 64, 0.25)


def test_jaccard_definition():
    """J(A,B) = |A n B| / |A u B| (page "Qwen4 in llama.cpp", section "QSA Is
    an Address-Selection Problem")."""
    from tests.helpers import jaccard
    assert jaccard([0, 1, 2, 5], [0, 2, 5, 7]) == pytest.approx(3 / 5)
    assert jaccard([0, 3], [0, 3]) == 1.0
    assert jaccard([0, -1, 4], [0, 4, -1]) == 1.0


# ------------------------------------------------------- quantized KV option
def test_fwht_is_the_sylvester_hadamard_product():
    """The rotation is the unnormalised Walsh-Hadamard transform: on integer
    inputs (exact in fp32) it equals the product with scipy's Sylvester
    Hadamard matrix, and applying it twice multiplies by n (H^2 = n I)."""
    import scipy.linalg
    g = np.random.RandomState(3)
    for n in (64, 128):
        x = g.randint(-50, 50, size=(5, n)).astype(np.float32)
        H = scipy.linalg.hadamard(n).astype(np.float64)
        assert np.array_equal(oracle.fwht_f32(x).astype(np.float64), x.astype(np.float64) @ H.T)
        assert np.array_equal(oracle.fwht_f32(oracle.fwht_f32(x)), n * x)


def test_e4m3_hand_values():
    """fp8 e4m3: 3 mantissa bits, bias 7, largest 448, subnormals m * 2^-9;
    nearest with ties to even, saturating."""
    cases = [
        (1.0, 0x38), (1.0625, 0x38),          # tie between 1 and 1.125: even (1)
        (1.1875, 0x3A),                        # tie between 1.125 and 1.25: even (1.25)
        (448.0, 0x7E), (460.0, 0x7E),          # 460 rounds to 448
        (470.0, 0x7E), (1e9, 0x7E),            # would round to 480 / overflow: saturates
        (-470.0, 0xFE),
        (2.0 ** -9, 0x01), (1.5 * 2.0 ** -9, 0x02),   # subnormal tie: even multiple
        (2.0 ** -10, 0x00),                    # tie between 0 and 2^-9: even (0)
        (2.0 ** -6, 0x08),                     # smallest normal
        (-3.3, 0xC5), (0.0, 0x00), (-0.0, 0x80),
    ]
    got = oracle.e4m3(np.array([c[0] for c in cases], dtype=np.float32))
    assert got.tolist() == [c[1] for c in cases]


def test_e4m3_matches_torch_within_range():
    """Inside the range where no saturation happens (|x| < 464), the codes
    are torch's fp32 -> float8_e4m3fn conversion; every finite code decodes
    to the value torch gives and encodes back to itself."""
    g = torch.Generator().manual_seed(9)
    x = torch.randn(50000, generator=g) * torch.exp2(torch.randint(-12, 9, (50000,), generator=g).float())
    x = x[x.abs() < 464]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3(x.numpy()), ref)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_value(codes), vals)
    assert np.array_equal(oracle.e4m3(vals.astype(np.float32)), codes)


def test_quantize_rows_fp8_scale_and_error():
    g = torch.Generator().manual_seed(10)
    X = bf16(torch.randn((40, 128), generator=g))
    codes, scales = oracle.quantize_kv_fp8(X)
    u = oracle.fwht_f32(f64(X).astype(np.float32))
    assert np.array_equal(scales, (np.abs(u).max(axis=1) / np.float32(448)).astype(np.float32))
    deq = oracle.e4m3_value(codes) * scales[:, None].astype(np.float64)
    # within half a code step (relative 2^-4 for normals) of the rotated row
    assert np.all(np.abs(deq - u) <= np.abs(u) * 2.0 ** -4 + scales[:, None] * 2.0 ** -10)
    # the largest element of each row becomes +-448
    am = np.abs(u).argmax(axis=1)
    assert np.all(np.abs(oracle.e4m3_value(codes[np.arange(40), am])) == 448.0)


def test_decode_fp8_equals_bf16_attention_on_walsh_rows():
    """Rows whose rotation has a single nonzero component are signed Walsh
    functions times c*s/n -- exact in bf16 -- and quantize without loss, so
    the quantized decode (rotated basis, output rotated back) must equal the
    pinned bf16 attention on the same K, V."""
    import scipy.linalg
    n, B, Hq, Hkv, T, L = 128, 2, 8, 2, 256, 200
    H = scipy.linalg.hadamard(n).astype(np.float64)
    g = np.random.RandomState(11)
    def walsh_rows(shape):
        # c = +-1.75 * 2^k: the rotated row's one nonzero is 16 c, its scale
        # 16 c / 448 = 2^k / 16 is a power of two, so the code 448 is exact
        j0 = g.randint(0, n, size=shape)
        c = g.choice([0.4375, 0.875, 1.75, 3.5, -0.875, -1.75], size=shape)
        return (c[..., None] * H[j0]) * 2.0 ** -3      # = c * 2^-3 * row j0 of H (exact in bf16)
    K = bf16(torch.from_numpy(walsh_rows((B, Hkv, T))).float())
    V = bf16(torch.from_numpy(walsh_rows((B, Hkv, T))).float())
    q = bf16(torch.randn((B, Hq, n), generator=torch.Generator().manual_seed(12)))
    ck, sk = oracle.quantize_kv_fp8(K)
    cv, sv = oracle.quantize_kv_fp8(V)
    assert np.allclose(oracle.fwht_f32(f64(K).astype(np.float32)),
                       oracle.e4m3_value(ck) * sk[..., None].astype(np.float64), rtol=0, atol=0)
    idx = np.array([[0, 1, 3, -1], [0, 2, 3, -1]] * B, dtype=np.int32).reshape(B, Hkv, 1, 4)
    sm = n ** -0.5
    o = oracle.decode_fp8(q, ck, sk, cv, sv, idx, L, sm)
    ref = oracle.attend(q.view(B, 1, Hq, n), K, V, idx, L - 1, 1, sm).reshape(B, Hq, n)
    assert np.abs(o - ref).max() < 1e-12


# ------------------------------------------------------ score aggregators
def _agg_case(seed, B=1, Tq=130, Hq=8, Hkv=2, d=64, q_pos0=64 * 6, qblk=64, nblk=10):
    g = torch.Generator().manual_seed(seed)
    Q = bf16(torch.randn((B, Tq, Hq, d), generator=g))
    K = bf16(torch.randn((B, Hkv, 64 * (nblk + 3), d), generator=g))
    Kc = oracle.compress_keys(K, 0, nblk + 2)
    return Q, K, Kc


def test_mean_aggregator_equals_pooled_query_scores():
    """Averaging the per-(head, token) logits equals scoring the pooled
    query (linearity); the two are computed independently."""
    Q, _, Kc = _agg_case(21)
    sm = 0.125
    for qblk, q_pos0 in ((64, 64 * 6), (1, 64 * 9 + 17)):
        Tq = Q.shape[1]
        s = oracle.block_scores(Q, Kc, Tq, q_pos0, qblk, sm, "mean")
        Qbar = oracle.pool_queries(Q, 2, qblk)
        ref = oracle.select(Qbar, Kc, Tq, q_pos0, qblk, 4, sm, want_scores=True)
        NB = Kc.shape[2]
        ref_s = ref["scores"].reshape(s.shape[:3] + (NB,))
        cand = ~np.isnan(ref_s)                          # candidates 1 .. D-1
        assert np.allclose(s[cand], ref_s[cand], rtol=0, atol=1e-12)
        # and the selection rule on the table reproduces the pooled selection
        sel = oracle.select_scores(s, 1, 2, Tq, q_pos0, qblk, 4)
        assert np.array_equal(sel["idx"].reshape(ref["idx"].shape), ref["idx"])


def test_max_aggregator_special_cases():
    """Max over tokens of the head mean: one token per row -> the mean;
    identical tokens in a block -> the mean; never below the mean; invariant
    under reordering the block's tokens and the group's heads."""
    Q, _, Kc = _agg_case(22)
    sm = 0.125
    Tq = Q.shape[1]
    one = oracle.block_scores(Q, Kc, Tq, 64 * 9, 1, sm, "max")
    assert np.array_equal(np.isnan(one), np.isnan(oracle.block_scores(Q, Kc, Tq, 64 * 9, 1, sm, "mean")))
    assert np.allclose(one, oracle.block_scores(Q, Kc, Tq, 64 * 9, 1, sm, "mean"), rtol=0, atol=1e-12,
                       equal_nan=True)
    same = Q.clone()
    same[:, :64] = Q[:, :1]
    mx = oracle.block_scores(same, Kc, Tq, 64 * 6, 64, sm, "max")[:, :, 0]
    mn = oracle.block_scores(same, Kc, Tq, 64 * 6, 64, sm, "mean")[:, :, 0]
    assert np.allclose(mx, mn, rtol=0, atol=1e-12, equal_nan=True)
    mx = oracle.block_scores(Q, Kc, Tq, 64 * 6, 64, sm, "max")
    mn = oracle.block_scores(Q, Kc, Tq, 64 * 6, 64, sm, "mean")
    ok = ~np.isnan(mx)
    assert np.all(mx[ok] >= mn[ok] - 1e-12) and np.mean(mx[ok] > mn[ok] + 1e-6) > 0.9
    perm = Q[:, torch.randperm(64, generator=torch.Generator().manual_seed(5))]
    perm = torch.cat([perm, Q[:, 64:]], 1)
    heads = torch.cat([Q[:, :, [3, 1, 0, 2]], Q[:, :, [7, 5, 6, 4]]], 2)
    for X in (perm, heads):
        assert np.allclose(oracle.block_scores(X, Kc, Tq, 64 * 6, 64, sm, "max")[:, :, 0], mx[:, :, 0],
                           rtol=0, atol=1e-12, equal_nan=True)


def test_softmax_sum_aggregator_pins():
    """Per-(head, token) softmax over the blocks before the diagonal, summed:
    the scores of a row add up to (heads x tokens); a vector added to every
    key leaves them unchanged (each softmax sees one constant shift); at zero
    temperature every block gets the same share, at a very low one each
    (head, token) votes for its best block; one head and token is the
    textbook softmax (scipy)."""
    import scipy.special
    Q, _, Kc = _agg_case(23)
    sm = 0.125
    Tq = Q.shape[1]
    s = oracle.block_scores(Q, Kc, Tq, 64 * 6, 64, sm, "softmax_sum")
    for i, ntok in ((0, 64), (1, 64), (2, 2)):
        D = (64 * 6 + min((i + 1) * 64, Tq) - 1) // 64
        row = s[0, 0, i]
        assert np.all(~np.isnan(row[:D])) and np.all(np.isnan(row[D:]))
        assert abs(row[:D].sum() - 4 * ntok) < 1e-9
    # every summary shifted by the same vector (in fp64: a shift of the bf16
    # keys would round)
    c = torch.randn(64, generator=torch.Generator().manual_seed(6)).double().numpy() * 3
    assert np.allclose(oracle.block_scores(Q, Kc + c, Tq, 64 * 6, 64, sm, "softmax_sum"), s, rtol=0,
                       atol=1e-10, equal_nan=True)
    flat = oracle.block_scores(Q, Kc, Tq, 64 * 6, 64, 0.0, "softmax_sum")
    D0 = 6 + 0   # row 0: diagonal block 6, blocks 0..5
    assert np.allclose(flat[0, 0, 0, :D0], 4 * 64 / D0, rtol=0, atol=1e-12)
    cold = oracle.block_scores(Q, Kc, Tq, 64 * 6, 64, 1e9, "softmax_sum")[0, 0, 0, :D0]
    z = np.einsum("thc,jc->thj", Q[0, :64, :4].double().numpy(), Kc[0, 0, :D0])
    votes = np.bincount(z.reshape(-1, D0).argmax(axis=1), minlength=D0)
    assert np.allclose(cold, votes, rtol=0, atol=1e-6)
    one = Q[:, :1, :2]                                           # one token, Hq = Hkv = 2 (G = 1)
    s1 = oracle.block_scores(one, Kc, 1, 64 * 7 + 3, 1, sm, "softmax_sum")[0, 1, 0, :7]
    zz = sm * (Kc[0, 1, :7] @ one[0, 0, 1].double().numpy())
    assert np.allclose(s1, scipy.special.softmax(zz), rtol=0, atol=1e-14)
