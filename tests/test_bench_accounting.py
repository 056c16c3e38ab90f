"""The benchmark's algorithmic work counts (the numerators of its roofline
fractions), checked on the CPU: the prefill FLOP count against a brute-force
count of the unmasked (query, key) pairs of the selected blocks on small
workloads, and both counts against the figures derived independently for
the benchmark's workloads (4*d*Hq FLOPs per pair; k*64*Hkv*d*2*2 bytes of
selected K+V per decode sequence)."""
import numpy as np
import pytest

import bench
import synthetic


def _pairs_brute(w):
    """Unmasked (query, key) pairs inside the selected blocks, counted one
    by one: a row keeps min(topk, D+1) blocks -- D itself plus D's
    predecessors, whichever they are (every non-diagonal block is wholly
    visible, so the choice does not change the count)."""
    total = 0
    for i in range(w.n_rows):
        t0, t1 = i * 64, min((i + 1) * 64, w.Tq)
        D = (w.q_pos0 + t1 - 1) // 64
        nsel = min(w.topk, D + 1)
        blocks = list(range(nsel - 1)) + [D]
        keys = np.concatenate([np.arange(64 * j, 64 * j + 64) for j in blocks])
        for t in range(t0, t1):
            total += int(np.count_nonzero(keys <= w.q_pos0 + t))
    return total * w.B


@pytest.mark.parametrize("kw", [
    dict(B=1, Tq=256, T_kv=256, q_pos0=0, Hq=8, Hkv=2, d=64, topk=4),
    dict(B=2, Tq=200, T_kv=64 * 40, q_pos0=64 * 30, Hq=16, Hkv=2, d=128, topk=16),
    dict(B=1, Tq=96, T_kv=64 * 8, q_pos0=64 * 5, Hq=16, Hkv=2, d=128, topk=64),
])
def test_prefill_flops_against_brute_force(kw):
    w = synthetic.custom(**kw)
    assert bench.prefill_flops(w) == 4.0 * w.d * w.Hq * _pairs_brute(w)


@pytest.mark.parametrize("name,gflop", [("prefill_128k", 2148.6), ("prefill_32k", 262.4), ("chunked_1m", 136.4)])
def test_prefill_flops_of_the_workloads(name, gflop):
    assert bench.prefill_flops(synthetic.CONFIGS[name]) / 1e9 == pytest.approx(gflop, rel=1e-3)


@pytest.mark.parametrize("name", ["decode_128k", "decode_262k"])
def test_decode_bytes_of_the_workloads(name):
    w = synthetic.CONFIGS[name]
    # every sequence keeps 64 full blocks minus the diagonal's unwritten tail
    D = w.q_pos0 // 64
    keys = 64 * (w.topk - 1) + (w.q_pos0 - 64 * D + 1)
    assert bench.decode_bytes(w) == w.B * w.Hkv * keys * w.d * 2 * 2
    # the diagonal block of these workloads is full, so the step moves 128 MiB
    assert bench.decode_bytes(w) == 128 << 20
