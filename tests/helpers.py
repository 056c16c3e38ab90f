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
