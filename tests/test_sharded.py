"""One long sequence whose cache is split over several GPUs by contiguous
block ranges (each rank: its blocks, their summaries and the whole Q).

CPU (oracle, fp64): every rank's top-m candidate lists, merged, give
exactly the selection of the unsharded cache, and attention over each
rank's selected blocks, merged by log-sum-exp, gives the unsharded output
to 1e-12 -- for uneven ranges, ranges that hold none of a row's candidates,
and through two gloo ranks exchanging their lists and partial outputs with
the package's all-gather helper.

GPU (one device, the ranks emulated one after another): the local-range
kernels (candidate lists, list merge, attention over the rank's own blocks,
partial merge) against the whole-cache kernels (indices bit for bit) and
against the oracle (selection rules, outputs within the tolerance); and the
orchestration class over a one-rank NCCL group.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synthetic


def _workload(seed=81, cache_blocks=150, Tq=192, topk=8, plant=0.05):
    # a chunked prefill: Tq new tokens after a cache of cache_blocks blocks
    return synthetic.custom(B=1, Tq=Tq, T_kv=64 * cache_blocks + Tq, q_pos0=64 * cache_blocks, qblk=64, Hq=8,
                            Hkv=2, d=64, topk=topk, seed=seed, plant="partner", plant_frac=plant)


def _local_idx(idx, lo, hi):
    """The rank's part of a selection: its blocks kept in order, -1 padded."""
    out = np.full_like(idx, -1)
    flat, dst = idx.reshape(-1, idx.shape[-1]), out.reshape(-1, idx.shape[-1])
    for r in range(flat.shape[0]):
        keep = [j for j in flat[r] if lo <= j < hi]
        dst[r, :len(keep)] = keep
    return out


def _sharded_oracle(w, x, ranges):
    """Each rank's lists and partial outputs (the rank sees only its own
    summaries), merged."""
    NB = w.T_kv // 64
    Kc = oracle.compress_keys(x["K"], 0, (w.q_pos0 + w.Tq) // 64)
    Qbar = oracle.pool_queries(x["Q"], w.Hkv, w.qblk)
    S, J = [], []
    for lo, hi in ranges:
        mine = np.zeros_like(Kc)
        mine[:, :, lo:hi] = Kc[:, :, lo:hi]
        s, j = oracle.select_shard(Qbar, mine, w.Tq, w.q_pos0, w.topk, w.sm_scale, lo, hi)
        S.append(s)
        J.append(j)
    idx = oracle.merge_shard_lists(np.stack(S), np.stack(J), w.Tq, w.q_pos0, w.topk)
    idx = idx.reshape(w.B, w.Hkv, w.n_rows, w.topk)
    Os, ls = [], []
    for lo, hi in ranges:
        O_r, lse_r = oracle.attend(x["Q"], x["K"], x["V"], _local_idx(idx, lo, hi), w.q_pos0, w.qblk, w.sm_scale,
                                   want_lse=True)
        Os.append(O_r)
        ls.append(lse_r)
    O, _ = oracle.merge_partials(np.stack(Os), np.stack(ls))
    assert NB >= ranges[-1][1]
    return idx, O


RANGES = {
    "two_halves": lambda nb: [(0, nb // 2), (nb // 2, nb)],
    "three_uneven": lambda nb: [(0, 7), (7, 100), (100, nb)],
    "sink_alone": lambda nb: [(0, 1), (1, 140), (140, nb)],
}


@pytest.mark.parametrize("split", sorted(RANGES))
def test_sharded_oracle_equals_unsharded(split):
    w = _workload()
    x = synthetic.generate(w)
    nb = w.T_kv // 64
    ranges = RANGES[split](nb)
    sel, O_ref = oracle.qsa_forward(x["Q"], x["K"], x["V"], w.Hkv, w.topk, q_pos0=w.q_pos0)
    idx, O = _sharded_oracle(w, x, ranges)
    assert np.array_equal(idx, sel["idx"])
    assert np.abs(O - O_ref).max() <= 1e-12


def test_merge_partials_closed_forms():
    rng = np.random.RandomState(3)
    O = rng.randn(4, 5, 8)
    lse = rng.randn(4, 5)
    # one part: itself
    O1, l1 = oracle.merge_partials(O[:1], lse[:1])
    assert np.allclose(O1, O[0], atol=1e-15) and np.allclose(l1, lse[0], atol=1e-15)
    # an empty part changes nothing
    O2, l2 = oracle.merge_partials(np.concatenate([O[:2], np.zeros((1, 5, 8))]),
                                   np.concatenate([lse[:2], np.full((1, 5), -np.inf)]))
    O3, l3 = oracle.merge_partials(O[:2], lse[:2])
    assert np.allclose(O2, O3, atol=1e-15) and np.allclose(l2, l3, atol=1e-15)
    # equal normalisers: the plain mean, lse + log(R)
    O4, l4 = oracle.merge_partials(O, np.zeros((4, 5)))
    assert np.allclose(O4, O.mean(axis=0), atol=1e-14) and np.allclose(l4, np.log(4), atol=1e-14)
    # all empty: zeros and -inf
    O5, l5 = oracle.merge_partials(np.zeros((2, 3, 4)), np.full((2, 3), -np.inf))
    assert (O5 == 0).all() and np.isneginf(l5).all()


def test_shard_ranges_cover_the_cache():
    import block_sparse_long_compress_b200 as qsa
    for nb, world in ((16448, 8), (10, 3), (5, 5)):
        r = qsa.shard_ranges(nb, world)
        assert r[0][0] == 0 and r[-1][1] == nb and len(r) == world
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        assert max(h - l for l, h in r) - min(h - l for l, h in r) <= 1
    with pytest.raises(ValueError):
        qsa.shard_ranges(2, 3)


# ------------------------------------------------------ two gloo ranks
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import block_sparse_long_compress_b200 as qsa
        w = _workload(seed=83)
        x = synthetic.generate(w)
        nb = w.T_kv // 64
        lo, hi = qsa.shard_ranges(nb, world)[rank]
        # this rank holds only its own blocks of K, V and of the summaries
        K = x["K"].clone()
        V = x["V"].clone()
        K[:, :, :64 * lo] = 0
        K[:, :, 64 * hi:] = 0
        V[:, :, :64 * lo] = 0
        V[:, :, 64 * hi:] = 0
        Kc = oracle.compress_keys(K, 0, (w.q_pos0 + w.Tq) // 64)
        Qbar = oracle.pool_queries(x["Q"], w.Hkv, w.qblk)
        s, j = oracle.select_shard(Qbar, Kc, w.Tq, w.q_pos0, w.topk, w.sm_scale, lo, hi)
        S = qsa.all_gather_rank_major(torch.from_numpy(s)).numpy()
        J = qsa.all_gather_rank_major(torch.from_numpy(j)).numpy()
        idx = oracle.merge_shard_lists(S, J, w.Tq, w.q_pos0, w.topk).reshape(w.B, w.Hkv, w.n_rows, w.topk)
        O_r, lse_r = oracle.attend(x["Q"], K, V, _local_idx(idx, lo, hi), w.q_pos0, w.qblk, w.sm_scale,
                                   want_lse=True)
        Os = qsa.all_gather_rank_major(torch.from_numpy(O_r)).numpy()
        ls = qsa.all_gather_rank_major(torch.from_numpy(lse_r)).numpy()
        O, _ = oracle.merge_partials(Os, ls)
        sel, O_ref = oracle.qsa_forward(x["Q"], x["K"], x["V"], w.Hkv, w.topk, q_pos0=w.q_pos0)
        out[rank] = (bool(np.array_equal(idx, sel["idx"])), float(np.abs(O - O_ref).max()))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_unsharded_path():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_gloo_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        for r in range(2):
            same, err = out[r]
            assert same, f"rank {r}: merged selection differs from the unsharded one"
            assert err <= 1e-12, (r, err)


# --------------------------------------------------------------- GPU
DEV = "cuda"


@pytest.mark.gpu
@pytest.mark.parametrize("split", ["two_halves", "three_uneven", "sink_alone"])
def test_sharded_kernels_match_whole_cache(split):
    import block_sparse_long_compress_b200 as qsa
    w = synthetic.custom(B=1, Tq=320, T_kv=64 * 700 + 320, q_pos0=64 * 700, qblk=64, Hq=16, Hkv=2, d=128, topk=16,
                         seed=85, plant="partner", plant_frac=0.05)
    x = synthetic.generate(w)
    Q, K, V = (x[k].to(DEV) for k in ("Q", "K", "V"))
    nb = w.T_kv // 64
    ranges = RANGES[split](nb)
    # the whole cache, as one GPU runs it
    run = qsa.QSAPrefill(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0, device=DEV, with_lse=True)
    run.precompress_cache(K)
    O_whole = run(Q, K, V).clone()
    assert qsa.device_status()[0] == "QSA_OK"
    Kc = run.Kc
    # every rank's lists, gathered rank-major
    nlists = max(qsa.select_local_lists(w.Tq, w.q_pos0, lo, hi) for lo, hi in ranges)
    lists = []
    for lo, hi in ranges:
        L = torch.full((w.B, w.Hkv, w.n_rows, nlists, 62), -5, dtype=torch.int64, device=DEV)
        qsa.score_select_local(Q, Kc[:, :, lo:hi].contiguous(), L, w.q_pos0, lo, hi, w.topk, w.sm_scale)
        lists.append(L)
    idx = torch.full_like(run.idx, -7)
    qsa.merge_select_lists(torch.stack(lists), idx, w.Tq, w.q_pos0)
    assert qsa.device_status()[0] == "QSA_OK"
    # the same fp32 scores and order: the whole-cache indices bit for bit
    assert torch.equal(idx, run.idx)
    # every rank attends over its own blocks; the partials merge
    Os, ls = [], []
    for lo, hi in ranges:
        Kl, Vl = K[:, :, 64 * lo:64 * hi].contiguous(), V[:, :, 64 * lo:64 * hi].contiguous()
        O_r = torch.full_like(Q, float("nan"))
        lse_r = torch.full((w.B, w.Tq, w.Hq), float("nan"), dtype=torch.float32, device=DEV)
        qsa.sparse_attn_prefill_local(Q, Kl, Vl, idx, O_r, lse_r, w.q_pos0, lo, hi, w.sm_scale)
        assert qsa.device_status()[0] == "QSA_OK"
        # the rank's partial against the oracle over the same blocks
        idx_r = _local_idx(idx.cpu().numpy(), lo, hi)
        O_ref_r, lse_ref_r = oracle.attend(x["Q"], x["K"], x["V"], idx_r, w.q_pos0, w.qblk, w.sm_scale,
                                           want_lse=True)
        empty = np.isneginf(lse_ref_r)
        got_lse = lse_r.cpu().numpy()
        assert np.array_equal(np.isneginf(got_lse), empty)
        assert np.abs(got_lse[~empty] - lse_ref_r[~empty]).max() <= 1e-3
        err = np.abs(O_r.float().cpu().numpy() - O_ref_r)
        assert err.max() <= 1e-2 and err.mean() <= 1e-3, (lo, hi, err.max(), err.mean())
        Os.append(O_r)
        ls.append(lse_r)
    O = torch.empty_like(Q)
    lse = torch.empty((w.B, w.Tq, w.Hq), dtype=torch.float32, device=DEV)
    qsa.merge_partials(torch.stack(Os), torch.stack(ls), O, lse)
    assert qsa.device_status()[0] == "QSA_OK"
    O_ref = oracle.attend(x["Q"], x["K"], x["V"], idx.cpu().numpy(), w.q_pos0, w.qblk, w.sm_scale)
    err = np.abs(O.float().cpu().numpy() - O_ref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
    assert np.abs(lse.cpu().numpy() - run.lse.cpu().numpy()).max() <= 1e-3
    print(f"sharded {split}: O max {err.max():.2e} mean {err.mean():.2e}; vs whole-cache "
          f"{(O.float() - O_whole.float()).abs().max().item():.2e}")


@pytest.mark.gpu
def test_sharded_class_over_a_one_rank_nccl_group():
    import block_sparse_long_compress_b200 as qsa
    w = _workload(seed=87)
    x = synthetic.generate(w)
    Q, K, V = (x[k].to(DEV) for k in ("Q", "K", "V"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    torch.distributed.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        nb = w.T_kv // 64
        Kc = torch.zeros((w.B, w.Hkv, nb, w.d), dtype=torch.float32, device=DEV)
        qsa.compress_keys(K, Kc, 0, (w.q_pos0 + w.Tq) // 64)
        sh = qsa.QSAShardedPrefill(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.topk, w.q_pos0, qsa.shard_ranges(nb, 1), 0,
                                   device=DEV)
        O = sh(Q, K, V, Kc)
        torch.cuda.synchronize()
        assert qsa.device_status()[0] == "QSA_OK"
        O_ref = oracle.attend(x["Q"], x["K"], x["V"], sh.idx.cpu().numpy(), w.q_pos0, w.qblk, w.sm_scale)
        err = np.abs(O.float().cpu().numpy() - O_ref)
        assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.gpu
def test_sharded_kernels_at_chunked_1m():
    """chunked_1m (4096 new tokens after a 1,048,576-token cache, top-64)
    split over 4 ranks, emulated one after another on one GPU: the merged
    indices equal the whole-cache path's bit for bit on all 128 rows, and the
    merged outputs of 512 tokens (the chunk's first and last query blocks
    and 384 drawn at random) are within the tolerance of the oracle."""
    import block_sparse_long_compress_b200 as qsa
    w = synthetic.CONFIGS["chunked_1m"]
    x = synthetic.generate(w, DEV)
    Q, K, V = x["Q"], x["K"], x["V"]
    nb = w.T_kv // 64
    run = qsa.QSAPrefill(w.B, w.Tq, w.Hq, w.Hkv, w.d, w.T_kv, w.topk, w.q_pos0, device=DEV)
    run.precompress_cache(K)
    run(Q, K, V)
    assert qsa.device_status()[0] == "QSA_OK"
    ranges = qsa.shard_ranges(nb, 4)
    nlists = max(qsa.select_local_lists(w.Tq, w.q_pos0, lo, hi) for lo, hi in ranges)
    lists = []
    for lo, hi in ranges:
        L = torch.empty((w.B, w.Hkv, w.n_rows, nlists, 62), dtype=torch.int64, device=DEV)
        qsa.score_select_local(Q, run.Kc[:, :, lo:hi].contiguous(), L, w.q_pos0, lo, hi, w.topk, w.sm_scale)
        lists.append(L)
    idx = torch.full_like(run.idx, -7)
    qsa.merge_select_lists(torch.stack(lists), idx, w.Tq, w.q_pos0)
    assert qsa.device_status()[0] == "QSA_OK"
    assert torch.equal(idx, run.idx)
    Os, ls = [], []
    for lo, hi in ranges:
        Kl, Vl = K[:, :, 64 * lo:64 * hi].contiguous(), V[:, :, 64 * lo:64 * hi].contiguous()
        O_r = torch.empty_like(Q)
        lse_r = torch.empty((w.B, w.Tq, w.Hq), dtype=torch.float32, device=DEV)
        qsa.sparse_attn_prefill_local(Q, Kl, Vl, idx, O_r, lse_r, w.q_pos0, lo, hi, w.sm_scale)
        Os.append(O_r)
        ls.append(lse_r)
        del Kl, Vl
    assert qsa.device_status()[0] == "QSA_OK"
    O = torch.empty_like(Q)
    qsa.merge_partials(torch.stack(Os), torch.stack(ls), O)
    assert qsa.device_status()[0] == "QSA_OK"
    rng = np.random.RandomState(29)
    toks = np.unique(np.concatenate([np.arange(64), np.arange(w.Tq - 64, w.Tq),
                                     rng.choice(np.arange(64, w.Tq - 64), 384, replace=False)]))
    O_ref = oracle.attend(Q.cpu(), K.cpu(), V.cpu(), idx.cpu().numpy(), w.q_pos0, w.qblk, w.sm_scale, tokens=toks)
    O_gpu = O.reshape(w.Tq, w.Hq, w.d)[torch.from_numpy(toks).to(DEV)].float().cpu().numpy()
    err = np.abs(O_gpu - O_ref)
    print(f"sharded chunked_1m (4 ranks): {err.size} outputs, max|err| {err.max():.3e} mean {err.mean():.3e}")
    assert err.max() <= 1e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
