"""The seeded input generators shared by the tests and the benchmark: the
same seed gives the same tensors, the planted structure is what the recipe
says, and the paged generators' block tables address every page at most
once and cover each sequence's length.  CPU only (small shapes)."""
import numpy as np
import torch

import synthetic


def test_generate_is_deterministic_and_bf16():
    w = synthetic.custom(B=2, Tq=96, T_kv=256, q_pos0=64, qblk=64, Hq=8, Hkv=2, d=64, topk=4, seed=5,
                         plant="partner", plant_frac=0.25)
    a, b = synthetic.generate(w), synthetic.generate(w)
    for k in ("Q", "K", "V"):
        assert a[k].dtype == torch.bfloat16 and torch.equal(a[k], b[k])
    assert a["planted"] == b["planted"]
    c = synthetic.generate(synthetic.Workload(**{**w.__dict__, "seed": 6}))
    assert not torch.equal(a["K"], c["K"])


def test_token_planting_recipe():
    """plant="token": int(frac * (D0 - 1)) blocks before the first token's
    diagonal per (sequence, group), sink excluded, each shifting its keys and
    the group's queries along one unit direction."""
    pos, frac, scale = 64 * 20 + 5, 0.25, 4.0
    w = synthetic.custom(B=2, Tq=2, T_kv=64 * 22, q_pos0=pos, qblk=1, Hq=8, Hkv=2, d=64, topk=4, seed=9,
                         plant="token", plant_frac=frac, plant_scale=scale)
    x = synthetic.generate(w)
    base = synthetic.generate(synthetic.Workload(**{**w.__dict__, "plant": "none"}))
    n_expected = int(frac * (pos // 64 - 1))
    for b in range(2):
        for g in range(2):
            js = sorted(j for (bb, gg, j, _) in x["planted"] if (bb, gg) == (b, g))
            assert len(js) == n_expected and len(set(js)) == n_expected
            assert all(1 <= j < pos // 64 for j in js)
            # only the planted blocks' keys changed
            dk = (x["K"][b, g].float() - base["K"][b, g].float()).view(-1, 64, 64)
            changed = [j for j in range(dk.shape[0]) if dk[j].abs().max() > 0]
            assert changed == js
    # every token's queries moved (the planted directions are added to the
    # group's heads of all of the row's tokens)
    dq = (x["Q"].float() - base["Q"].float())
    assert all(dq[:, t].abs().max() > 0 for t in range(w.Tq))


def test_paged_decode_tables_and_lengths():
    x = synthetic.paged_decode(B=4, min_len=100, max_len=1000, Hq=8, Hkv=2, d=64, seed=3)
    table = x["block_table"].numpy()
    assert table.shape == (4, x["max_blocks"]) and x["max_blocks"] == (1000 + 63) // 64
    assert len(np.unique(table)) == table.size                       # every page at most once
    assert table.min() >= 0 and table.max() < x["K_pages"].shape[0]
    lens = x["seq_lens"].numpy()
    assert lens.min() >= 100 and lens.max() <= 1000 and x["max_len"] == lens.max()
    y = synthetic.paged_decode(B=4, min_len=100, max_len=1000, Hq=8, Hkv=2, d=64, seed=3)
    assert torch.equal(x["K_pages"], y["K_pages"]) and np.array_equal(table, y["block_table"].numpy())


def test_paged_prefill_positions():
    x = synthetic.paged_prefill(B=3, Tq=128, min_pos=640, max_pos=3200, Hq=8, Hkv=2, d=64, seed=4)
    q_pos = x["q_pos"].numpy()
    assert np.all(q_pos % 64 == 0) and q_pos.min() >= 640 and q_pos.max() <= 3200
    assert x["max_blocks"] * 64 >= q_pos.max() + 128                   # the chunk fits after the cache
    table = x["block_table"].numpy()
    assert len(np.unique(table)) == table.size
