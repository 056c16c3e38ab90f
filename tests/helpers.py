"""Comparison helpers shared by the tests (no method arithmetic)."""
import numpy as np


def jaccard(a, b):
    """Set overlap J(A, B) = |A n B| / |A u B| of two selections; -1 padding
    is ignored (page "Qwen4 in llama.cpp: Dissecting PR #27742", section
    "QSA Is an Address-Selection Problem, Not a New Attention Equation")."""
    A = {int(x) for x in a if x >= 0}
    B = {int(x) for x in b if x >= 0}
    if not A and not B:
        return 1.0
    return len(A & B) / len(A | B)


def to_bits(t):
    """torch bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------- GPU-vs-oracle checks
def check_selection(idx_gpu, sel_ref, scores_ref, rows_D, topk, gap_tol=1e-3, valid_tol=1e-5):
    """idx_gpu, sel_ref['idx']: [nrows, topk]; scores_ref: [nrows, NB]."""
    idx_ref, gap = sel_ref["idx"], sel_ref["gap"]
    n = len(idx_gpu)
    exact = gap > gap_tol
    assert np.array_equal(idx_gpu[exact], idx_ref[exact]), "indices differ on a clear-gap row"
    jac = []
    for r in range(n):
        row = [int(j) for j in idx_gpu[r] if j >= 0]
        D = rows_D[r]
        assert row == sorted(set(row)) and row[0] == 0 and (D == 0 or row[-1] == D)
        assert all(j == -1 for j in idx_gpu[r][len(row):])
        assert len(row) == int(np.sum(idx_ref[r] >= 0))
        chosen = [j for j in row if 0 < j < D]
        cand = np.arange(1, D)
        unchosen = np.setdiff1d(cand, chosen)
        if chosen and len(unchosen):
            s = scores_ref[r]
            assert s[chosen].min() >= s[unchosen].max() - valid_tol, f"row {r}: not a valid top-m"
        jac.append(jaccard(idx_gpu[r], idx_ref[r]))
    return float(exact.mean()), float(np.mean(jac))


def check_out(O_gpu, O_ref, max_tol=1e-2, mean_tol=1e-3):
    err = np.abs(np.asarray(O_gpu, dtype=np.float64) - O_ref)
    assert np.isfinite(err).all()
    assert err.max() <= max_tol and err.mean() <= mean_tol, (err.max(), err.mean())
    return err.max(), err.mean()


def rows_diag(w):
    NR = w.n_rows
    D = []
    for b in range(w.B):
        for g in range(w.Hkv):
            for i in range(NR):
                D.append((w.q_pos0 + min((i + 1) * w.qblk, w.Tq) - 1) // 64)
    return D
