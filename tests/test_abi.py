"""Host-side checks of the C ABI (no GPU needed): the library builds and
loads, exports every entry point include/qsa.h declares, and rejects bad
arguments before launching anything."""
import ctypes
import re
import subprocess

import pytest
import torch

import block_sparse_long_compress_b200 as qsa


def test_exports_every_declared_symbol():
    declared = qsa.declared_symbols()
    assert len(declared) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", qsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (qsa_\w+)", out))
    assert set(declared) <= exported, set(declared) - exported
    for name in declared:
        assert hasattr(qsa.lib(), name)


def test_noalloc_scratch_size_matches_header():
    text = open(qsa.HEADER_PATH).read()
    m = re.search(r"#define QSA_SELECT_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m, "QSA_SELECT_SCRATCH_BYTES not found"
    assert qsa.SELECT_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_status_strings_and_last_error():
    lib = qsa.lib()
    for code, name in qsa.STATUS.items():
        assert lib.qsa_status_string(code).decode() == name
    assert lib.qsa_status_string(99).decode() == "QSA_ERR_UNKNOWN"


def test_workspace_sizes_are_host_only():
    # chunked selection (one 1M-token row per group) needs partial-key space
    big = qsa.score_select_workspace(1, 16, 2, 4096, 1048576, 64, 128, 64)
    small = qsa.score_select_workspace(1, 16, 2, 4096, 0, 64, 128, 64)
    assert big > small > 0
    assert qsa.score_select_workspace(1, 16, 2, 4096, 0, 7, 128, 64) == 0   # bad qblk
    # per-token selection (decode) is one launch whose chunks merge in distributed
    # shared memory: no workspace up to 8 x 8192 candidates, the chunked path beyond
    assert qsa.score_select_workspace(32, 16, 2, 1, 262143, 1, 128, 64) == 0
    assert qsa.score_select_workspace(1, 16, 2, 1, 64 * 70000, 1, 128, 64) > 0
    # decode merges its split-K partials in distributed shared memory: no workspace
    assert qsa.decode_workspace(32, 16, 2, 128, 64) == 0


def test_argument_checks_return_before_launch():
    lib = qsa.lib()
    P = ctypes.c_void_p
    fake = P(0x1000)       # never dereferenced: checks fail first
    odd = P(0x1008)
    # null pointer
    assert lib.qsa_compress_keys(None, fake, 1, 2, 128, 128, 0, 2, None) == 1
    assert b"null" in lib.qsa_last_error()
    # block range outside the cache
    assert lib.qsa_compress_keys(fake, fake, 1, 2, 128, 128, 0, 3, None) == 1
    # unsupported head dim
    assert lib.qsa_compress_keys(fake, fake, 1, 2, 128, 96, 0, 2, None) == 2
    # misaligned
    assert lib.qsa_compress_keys(odd, fake, 1, 2, 128, 128, 0, 2, None) == 1
    # score/select: q_pos0 not block aligned in prefill mode, topk too large, no workspace
    args = lambda **k: dict(dict(Q=fake, Kc=fake, idx=fake, B=1, Hq=16, Hkv=2, Tq=128, q_pos0=0,
                                 qblk=64, T=1024, d=128, topk=16, ws=fake, wsb=1 << 30), **k)

    def ss(a):
        return lib.qsa_score_select(a["Q"], a["Kc"], a["idx"], a["B"], a["Hq"], a["Hkv"], a["Tq"],
                                    a["q_pos0"], a["qblk"], a["T"], a["d"], a["topk"], 0.088,
                                    a["ws"], a["wsb"], None)
    assert ss(args(q_pos0=32)) == 1
    assert ss(args(topk=65)) == 2
    assert ss(args(topk=1)) == 2
    assert ss(args(qblk=16)) == 2
    assert ss(args(Tq=2000)) == 1          # queries past the cache
    assert ss(args(ws=None)) == 6
    assert ss(args(wsb=16)) == 6
    # prefill: unsupported group size, bad position
    pf = lambda Hq=16, q_pos0=0, d=128: lib.qsa_sparse_attn_prefill(
        fake, fake, fake, fake, fake, None, 1, Hq, 2, 128, q_pos0, 1024, d, 16, 0.088, None)
    assert pf(Hq=12) == 2
    assert pf(q_pos0=64 * 3 + 1) == 1
    assert pf(d=256) == 2
    # decode: L beyond the cache, small workspace
    dc = lambda L=1000, wsb=1 << 30: lib.qsa_decode(fake, fake, fake, fake, fake, 4, 16, 2, L,
                                                    1024, 128, 8, 0.088, fake, wsb, None)
    assert dc(L=2000) == 1
    assert lib.qsa_decode(fake, fake, fake, fake, fake, 40000, 16, 2, 64, 64, 128, 8, 0.088,
                          None, 0, None) == 2          # too many (sequence, group) rows
    # rotated fp8 cache: rows are 128 wide, scales 4-byte aligned, no negative count
    assert lib.qsa_quantize_kv_fp8(fake, fake, fake, 4, 64, None) == 2
    assert lib.qsa_quantize_kv_fp8(fake, fake, P(0x1002), 4, 128, None) == 1
    assert lib.qsa_quantize_kv_fp8(fake, fake, fake, -1, 128, None) == 1
    assert lib.qsa_quantize_kv_fp8(fake, fake, fake, 0, 128, None) == 0      # nothing to do
    d8 = lambda Hq=16, L=1000, d=128, topk=8, ks=fake: lib.qsa_decode_fp8(
        fake, fake, ks, fake, fake, fake, fake, 4, Hq, 2, L, 1024, d, topk, 0.088, None)
    assert d8(d=64) == 2
    assert d8(Hq=12) == 2
    assert d8(L=2000) == 1
    assert d8(topk=65) == 2
    assert d8(ks=odd) == 1
    assert d8(ks=None) == 1
    # per-token selection with an aggregator: unknown aggregator, ragged with
    # several tokens, a group of more than 8 heads
    ag = lambda agg=2, Tq=1, sl=None, Hq=16, Hkv=2, pos=1000: lib.qsa_score_select_token_agg(
        fake, fake, sl, fake, 4, Hq, Hkv, Tq, pos, 64, 128, 16, 0.088, agg, None)
    assert ag(agg=3) == 1
    assert ag(Tq=2, sl=fake) == 1
    assert ag(Hq=32, Hkv=2) == 2
    assert ag(agg=2, Tq=40, pos=4080) == 1   # queries past the summaries' capacity (64 blocks)
    # prefill rows, max aggregator: d must be 128, q_pos0 block aligned, a workspace
    pm = lambda d=128, pos=0, ws=fake, wsb=1 << 30, Hq=16, agg=1: lib.qsa_score_select_prefill_agg(
        fake, fake, fake, 1, Hq, 2, 128, pos, 1024, d, 16, 0.088, agg, ws, wsb, None)
    assert pm(d=64) == 2
    assert pm(pos=32) == 1
    assert pm(Hq=12) == 2
    assert pm(ws=None) == 6
    assert pm(agg=0) == 2                  # the mean has its own entry
    assert pm(agg=7) == 1
    wmax = lib.qsa_score_select_prefill_agg_workspace(1, 16, 2, 128, 0, 1024, 128, 16, 1)
    wsum = lib.qsa_score_select_prefill_agg_workspace(1, 16, 2, 128, 0, 1024, 128, 16, 2)
    assert wmax >= 2 * 2 * 16 * 4 and wsum >= wmax + 2 * 2 * 64 * 8 * 2 * 4
    # self-test limit out of range
    assert lib.qsa_selftest_wait_timeout(0, None) == 1


def test_product_path_has_no_oracle_dependency():
    """The package must not import or reach the oracle."""
    import os
    pkg = os.path.dirname(qsa.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f)).read()
                assert "oracle" not in text.lower(), f


def test_build_refuses_a_prefill_kernel_below_its_register_split():
    """The prefill kernel's setmaxnreg split assumes its launch register
    count; the build checks the compiler's report and refuses anything else."""
    import importlib.util
    import os
    spec = importlib.util.spec_from_file_location(
        "qsa_build", os.path.join(os.path.dirname(__file__), "..", "block_sparse_long_compress_b200",
                                  "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    ok = ("ptxas info    : Compiling entry function '_ZN3qsa26sparse_attn_prefill_kernelILi128ELi8EE'\n"
          f"ptxas info    : Used {build.PREFILL_LAUNCH_REGS} registers, used 1 barriers\n"
          "ptxas info    : Compiling entry function '_ZN3qsa13decode_kernelILi128ELi8EE'\n"
          "ptxas info    : Used 107 registers\n")
    build._check_registers(ok)
    with pytest.raises(RuntimeError):
        build._check_registers(ok.replace(f"Used {build.PREFILL_LAUNCH_REGS}", "Used 160"))


def test_binding_refuses_host_tensors_and_wrong_types():
    """The Python wrappers check device, dtype and shape before any call into
    the library (no GPU needed to see them refuse)."""
    bf = torch.bfloat16
    with pytest.raises(ValueError):
        qsa.quantize_kv_fp8(torch.zeros((2, 64), dtype=bf))            # rows must be 128 wide
    with pytest.raises(TypeError):
        qsa.quantize_kv_fp8(torch.zeros((2, 128), dtype=bf))           # a host tensor
    q = torch.zeros((1, 8, 128), dtype=bf)
    codes = torch.zeros((1, 2, 64, 128), dtype=torch.uint8)
    scales = torch.zeros((1, 2, 64), dtype=torch.float32)
    idx = torch.zeros((1, 2, 1, 4), dtype=torch.int32)
    with pytest.raises(TypeError):
        qsa.decode_fp8(q, codes, scales, codes, scales, idx, q.clone(), 64)
    with pytest.raises(ValueError):
        qsa.score_select_token_agg(torch.zeros((1, 1, 8, 128), dtype=bf), torch.zeros((1, 2, 4, 128)),
                                   idx, 4, 100, "median")
    with pytest.raises(ValueError):
        qsa.score_select_prefill_agg(torch.zeros((1, 64, 8, 128), dtype=bf), torch.zeros((1, 2, 4, 128)),
                                     torch.zeros((1, 2, 1, 4), dtype=torch.int32), 4, 0, "mean")
    with pytest.raises(TypeError):
        qsa.score_select_prefill_agg(torch.zeros((1, 64, 8, 128), dtype=bf), torch.zeros((1, 2, 4, 128)),
                                     torch.zeros((1, 2, 1, 4), dtype=torch.int32), 4, 0, "max")


def test_host_pipeline_checks_the_shape_before_touching_a_device():
    """qsa_prefill_pipeline_create validates on the host first: bad shapes
    return INVALID_ARG / UNSUPPORTED and leave *out NULL (this runs without
    a GPU, so any CUDA call would fail instead)."""
    lib = qsa.lib()
    h = ctypes.c_void_p(0)
    cases = [
        ((1, 16, 2, 256, 32, 1024, 128, 32, 0.088), 1),    # q_pos0 not a multiple of 64
        ((1, 16, 2, 256, 896, 1024, 128, 32, 0.088), 1),   # q_pos0 + Tq > T_kv_max
        ((1, 16, 3, 256, 0, 1024, 128, 32, 0.088), 1),     # Hq % Hkv != 0
        ((1, 16, 2, 256, 0, 1000, 128, 32, 0.088), 1),     # T_kv_max not a multiple of 64
        ((1, 16, 2, 256, 0, 1024, 96, 32, 0.088), 2),      # d unsupported
        ((1, 12, 2, 256, 0, 1024, 128, 32, 0.088), 2),     # G = 6 unsupported
        ((1, 16, 2, 256, 0, 1024, 128, 65, 0.088), 2),     # topk > 64
        ((1, 16, 2, 256, 0, 1024, 128, 32, 0.0), 1),       # sm_scale <= 0
    ]
    for (B, Hq, Hkv, Tq, q0, T, d, topk, sc), want in cases:
        rc = lib.qsa_prefill_pipeline_create(ctypes.byref(h), B, Hq, Hkv, Tq, q0, T, d, topk,
                                             ctypes.c_float(sc))
        assert rc == want, ((B, Hq, Hkv, Tq, q0, T, d, topk, sc), rc)
        assert not h.value
    assert lib.qsa_prefill_pipeline_create(None, 1, 16, 2, 256, 0, 1024, 128, 32, ctypes.c_float(0.088)) == 1
    assert lib.qsa_prefill_pipeline_submit(None, None, None, None, None) == 1
    assert lib.qsa_prefill_pipeline_synchronize(None) == 1
    assert lib.qsa_prefill_pipeline_destroy(None) == 0

