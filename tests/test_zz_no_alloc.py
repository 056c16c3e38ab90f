"""Allocation-free block selection (qsa_score_select_noalloc).

Some callers cannot allocate device memory at the point where they run the
selection: a custom operator or plug-in inside a host inference engine whose
memory planner owns the whole device (side allocations are forbidden or
would break its accounting), or a runtime with no allocator handle at the
call site.  For them the library carries a fixed static scratch buffer and
this entry point uses it instead of a caller workspace.

The test calls the new entry point through the C ABI and checks that two
calls in a row reproduce the selection of the workspace-taking entry point
exactly (block indices are integer results, compared bit for bit).  Every
case needs scratch memory, so every case reads and writes the static buffer:
  * prefill_tiny: the scratch holds the pooled queries and the rows' score
    table;
  * prefill_long_rows: rows of 2999 candidates, each selected whole from
    the score table (a larger table);
  * decode_long_rows: per-token rows of 69999 candidates (a 4.48M-token
    context), too long for the one-launch cluster path: the scratch holds
    the pooled queries and each chunk's top-m list, merged by a second
    kernel.
The summaries of the two larger cases are drawn directly (the comparison is
between two entry points on the same inputs, not against the oracle).
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

# (name, workload keywords, compress the drawn keys (True) or draw summaries)
CASES = [
    ("prefill_tiny", None, True),
    ("prefill_long_rows", dict(B=1, Tq=128, T_kv=64 * 3002, q_pos0=64 * 3000, qblk=64, Hq=16, Hkv=2,
                             d=128, topk=16), False),
    ("decode_long_rows", dict(B=1, Tq=1, T_kv=64 * 70001, q_pos0=64 * 70001 - 1, qblk=1, Hq=16,
                              Hkv=2, d=128, topk=64), False),
]


def _noalloc(qsa, Q, Kc, idx, w):
    fn = qsa.lib().qsa_score_select_noalloc
    return fn(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(Kc.data_ptr()),
              ctypes.c_void_p(idx.data_ptr()), w.B, w.Hq, w.Hkv, w.Tq, w.q_pos0, w.qblk,
              Kc.shape[2] * 64, w.d, w.topk, ctypes.c_float(w.sm_scale),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _inputs(w, compress):
    import block_sparse_long_compress_b200 as qsa
    if compress:
        x = synthetic.generate(w)
        Q, K = x["Q"].cuda(), x["K"].cuda()
        Kc = torch.zeros((w.B, w.Hkv, w.T_kv // 64, w.d), dtype=torch.float32, device="cuda")
        qsa.compress_keys(K, Kc)
        return Q, Kc
    g = torch.Generator(device="cuda")
    g.manual_seed(w.seed)
    Q = torch.randn((w.B, w.Tq, w.Hq, w.d), generator=g, device="cuda").to(torch.bfloat16)
    # summaries of 64 N(0,1) keys have a spread of 1/8 per component
    Kc = torch.randn((w.B, w.Hkv, w.T_kv // 64, w.d), generator=g, device="cuda") / 8
    return Q, Kc


@pytest.mark.parametrize("name,kw,compress", CASES, ids=[c[0] for c in CASES])
def test_noalloc_selection_matches_workspace_entry_point(name, kw, compress):
    import block_sparse_long_compress_b200 as qsa
    w = synthetic.CONFIGS["tiny_prefill_1k"] if kw is None else synthetic.custom(seed=71, **kw)
    Q, Kc = _inputs(w, compress)
    need = qsa.score_select_workspace(w.B, w.Hq, w.Hkv, w.Tq, w.q_pos0, w.qblk, w.d, w.topk)
    qbar_bytes = -(-w.B * w.Hkv * w.n_rows * w.d * 4 // 256) * 256
    assert need > 0, "this case must use the scratch buffer"
    if name != "prefill_tiny":
        assert need > qbar_bytes, "this case must also keep a score table or chunk lists in the scratch"
    assert need <= qsa.SELECT_SCRATCH_BYTES
    shape = (w.B, w.Hkv, w.n_rows, w.topk)
    ref = torch.full(shape, -7, dtype=torch.int32, device="cuda")
    qsa.score_select(Q, Kc, ref, w.topk, w.q_pos0, w.qblk, w.sm_scale)
    assert qsa.device_status()[0] == "QSA_OK"
    assert (ref[..., 0] == 0).all() and (ref >= -1).all()
    for call in range(2):
        out = torch.full(shape, -7, dtype=torch.int32, device="cuda")
        rc = _noalloc(qsa, Q, Kc, out, w)
        assert rc == 0, qsa.lib().qsa_last_error()
        assert qsa.device_status()[0] == "QSA_OK"
        assert torch.equal(out, ref), f"call {call}: selection differs"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import block_sparse_long_compress_b200 as qsa
    # 8 x 131072 prefill rows would need ~8 MiB of pooled queries: refused on the host
    need = qsa.score_select_workspace(8, 16, 2, 131072, 0, 64, 128, 32)
    assert need > qsa.SELECT_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = qsa.lib().qsa_score_select_noalloc(p, p, p, 8, 16, 2, 131072, 0, 64, 131072, 128, 32,
                                           ctypes.c_float(0.088), None)
    assert rc == 6
    assert b"static buffer" in qsa.lib().qsa_last_error()
