"""The host-buffer prefill pipeline (qsa_prefill_pipeline_*): steps fed
from pinned host memory through the library's own streams and device
buffers give, step for step, the outputs of the device-pointer path on the
same inputs (the same kernels: compared bit for bit), with neighbouring
steps in flight at once and the two buffer sets reused."""
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [
    ("g8_ragged", dict(B=2, Tq=300, T_kv=64 * 40, q_pos0=64 * 30, Hq=16, Hkv=2, d=128, topk=16)),
    ("g4_d64", dict(B=1, Tq=512, T_kv=1024, q_pos0=512, Hq=8, Hkv=2, d=64, topk=8)),
], ids=["g8_ragged", "g4_d64"])
def test_pipeline_steps_match_the_device_path(name, kw):
    import block_sparse_long_compress_b200 as qsa
    ws = [synthetic.custom(seed=90 + s, **kw) for s in range(2)]
    w = ws[0]
    xs = [synthetic.generate(v) for v in ws]     # two different inputs, alternated
    ref = []
    for x in xs:
        run = qsa.QSAPrefill(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0, device="cuda")
        Q, K, V = x["Q"].cuda(), x["K"].cuda(), x["V"].cuda()
        run.precompress_cache(K)
        ref.append(run(Q, K, V).cpu())
    assert qsa.device_status()[0] == "QSA_OK"
    host = [{k: x[k].contiguous().pin_memory() for k in ("Q", "K", "V")} for x in xs]
    outs = [torch.empty((w.B, w.Tq, w.Hq, w.d), dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    pipe = qsa.PrefillHostPipeline(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0)
    for k in range(5):
        h = host[k % 2]
        pipe.submit(h["Q"], h["K"], h["V"], outs[k])
    pipe.synchronize()
    assert qsa.device_status()[0] == "QSA_OK"
    for k in range(5):
        assert torch.equal(outs[k], ref[k % 2]), f"step {k} differs from the device path"
    pipe.close()


def test_pipeline_refuses_pageable_and_misshaped_host_buffers():
    import block_sparse_long_compress_b200 as qsa
    w = synthetic.custom(B=1, Tq=128, T_kv=512, q_pos0=0, Hq=16, Hkv=2, d=128, topk=8, seed=3)
    pipe = qsa.PrefillHostPipeline(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0)
    Q = torch.zeros((1, 128, 16, 128), dtype=torch.bfloat16)
    KV = torch.zeros((1, 2, 512, 128), dtype=torch.bfloat16).pin_memory()
    O = torch.zeros((1, 128, 16, 128), dtype=torch.bfloat16).pin_memory()
    with pytest.raises(ValueError, match="pinned"):
        pipe.submit(Q, KV, KV, O)                  # pageable Q
    with pytest.raises(ValueError, match="contiguous"):
        pipe.submit(O, KV[:, :, :256], KV, O)      # wrong K shape
    with pytest.raises(TypeError):
        pipe.submit(O.cuda(), KV, KV, O)           # a device tensor
    pipe.close()
