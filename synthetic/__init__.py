"""Seeded synthetic QSA workloads -- shared by the tests, the smoke check and
the benchmark.  This module only draws random numbers and plants structure;
it holds none of the method's arithmetic (no compression, scoring,
selection or attention).

Workloads mirror the long-context regime the pages discuss (contexts of 32K
to 1M tokens, 2 KV heads per QSA layer): page "Qwen3.8 Flash Next VRAM"
(vramcalculator.com), section "What It Needs" (12 of 48 layers are QSA
layers with 2 KV heads), and page "Qwen4 in llama.cpp: Dissecting PR
#27742", section "Why Short-Context Tests Can Lie" (4K ... 262K contexts).
No public dataset is involved; Q, K and V stand for post-RoPE activations.

Recipe (every workload):
  1. Q, K, V are drawn N(0, 1) in fp32 from ``torch.Generator(device)``
     seeded with the workload seed, in the order Q, K, V (K and V of a
     decode cache are drawn one sequence at a time, K then V).
  2. Planting parameters (block choices, partners, unit directions) are
     drawn from a separate CPU generator seeded with seed + 7.
  3. The planted offsets are added in fp32 and every tensor is rounded to
     bf16 once.
Layouts: Q [B, Tq, Hq, d]; K, V [B, Hkv, T_kv, d]; query head h belongs to
KV group h // (Hq // Hkv).
"""
import math
from dataclasses import dataclass, field

import torch

BLOCK = 64


@dataclass
class Workload:
    name: str
    B: int
    Tq: int
    T_kv: int
    Hq: int
    Hkv: int
    d: int
    topk: int
    q_pos0: int
    qblk: int
    seed: int
    plant: str = "none"          # "none" | "qhat" | "partner" | "token"
    plant_frac: float = 0.0
    plant_scale: float = 1.0
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def n_rows(self) -> int:
        return -(-self.Tq // self.qblk)

    @property
    def mode(self) -> str:
        return "decode" if self.qblk == 1 else "prefill"


# The five workload shapes, plus the 128K-context decode variant.
CONFIGS = {
    "tiny_prefill_1k": Workload(
        "tiny_prefill_1k", B=1, Tq=1024, T_kv=1024, Hq=8, Hkv=2, d=64, topk=4,
        q_pos0=0, qblk=BLOCK, seed=1001, plant="qhat", plant_scale=0.5,
        description="batch 1, T=1024, 8 q heads / 2 KV heads, d=64, block 64, top-k 4; "
                    "keys of 2 earlier blocks per query block get +0.5*qhat"),
    "prefill_32k": Workload(
        "prefill_32k", B=1, Tq=32768, T_kv=32768, Hq=16, Hkv=2, d=128, topk=16,
        q_pos0=0, qblk=BLOCK, seed=1002, plant="partner", plant_frac=0.10,
        description="batch 1, T=32768, 16 q heads / 2 KV heads, d=128, block 64, top-k 16; "
                    "10% of key blocks planted with a direction shared by one later query block"),
    "prefill_128k": Workload(
        "prefill_128k", B=1, Tq=131072, T_kv=131072, Hq=16, Hkv=2, d=128, topk=32,
        q_pos0=0, qblk=BLOCK, seed=1003, plant="partner", plant_frac=0.05,
        description="batch 1, T=131072, 16 q heads / 2 KV heads, d=128, block 64, top-k 32, "
                    "causal; 5% planted key blocks"),
    "decode_262k": Workload(
        "decode_262k", B=32, Tq=1, T_kv=262144, Hq=16, Hkv=2, d=128, topk=64,
        q_pos0=262143, qblk=1, seed=1004,
        description="decode: 32 single-token queries, each over its own 262144-token cache, "
                    "16 q heads / 2 KV heads, d=128, block 64, top-k 64 per token"),
    "decode_128k": Workload(
        "decode_128k", B=32, Tq=1, T_kv=131072, Hq=16, Hkv=2, d=128, topk=64,
        q_pos0=131071, qblk=1, seed=1006,
        description="decode at 128K context: 32 single-token queries over 131072-token caches"),
    "chunked_1m": Workload(
        "chunked_1m", B=1, Tq=4096, T_kv=1048576 + 4096, Hq=16, Hkv=2, d=128, topk=64,
        q_pos0=1048576, qblk=BLOCK, seed=1005, plant="partner", plant_frac=0.02,
        description="chunked prefill: 4096 new query tokens attending to a 1048576-token "
                    "cache plus themselves; block 64, top-k 64; 2% planted blocks"),
}


def custom(name="custom", *, B=1, Tq=256, T_kv=None, Hq=8, Hkv=2, d=64, topk=4,
           q_pos0=None, qblk=BLOCK, seed=7, plant="none", plant_frac=0.0,
           plant_scale=1.0) -> Workload:
    """A small ad-hoc workload (tests).  By default the queries are the last
    Tq positions of the cache."""
    if T_kv is None:
        T_kv = Tq if q_pos0 is None else q_pos0 + Tq
    if q_pos0 is None:
        q_pos0 = T_kv - Tq
    return Workload(name, B=B, Tq=Tq, T_kv=T_kv, Hq=Hq, Hkv=Hkv, d=d, topk=topk,
                    q_pos0=q_pos0, qblk=qblk, seed=seed, plant=plant,
                    plant_frac=plant_frac, plant_scale=plant_scale)


def _unit(gen, d):
    u = torch.randn(d, generator=gen, dtype=torch.float32)
    return u / u.norm()


def generate(w: Workload, device="cpu"):
    """Draw Q, K, V for workload ``w`` on ``device`` (bf16).

    Returns a dict with Q, K, V and ``planted`` (list of (b, g, key block,
    query row) tuples, for statistics only)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    Q = torch.randn((w.B, w.Tq, w.Hq, w.d), generator=gen, device=dev, dtype=torch.float32)
    big = w.B * w.Hkv * w.T_kv * w.d > (1 << 28)
    if big:
        # one sequence at a time to bound the fp32 staging memory
        K = torch.empty((w.B, w.Hkv, w.T_kv, w.d), device=dev, dtype=torch.bfloat16)
        V = torch.empty_like(K)
        kv_f32 = None
    else:
        Kf = torch.randn((w.B, w.Hkv, w.T_kv, w.d), generator=gen, device=dev, dtype=torch.float32)
        Vf = torch.randn((w.B, w.Hkv, w.T_kv, w.d), generator=gen, device=dev, dtype=torch.float32)
        kv_f32 = (Kf, Vf)

    G = w.Hq // w.Hkv
    pgen = torch.Generator(device="cpu")
    pgen.manual_seed(w.seed + 7)
    planted = []
    adds_k = []   # (b, g, j, vector)
    adds_q = []   # (b, g, row, vector)
    NB_kv = w.T_kv // BLOCK
    if w.plant == "qhat":
        # Per query block i >= 2 of each group: min(2, i-1) distinct earlier
        # blocks in [1, i-1] receive plant_scale * qhat on all their keys,
        # qhat being the unit direction of the block's summed queries over
        # the group's heads (drawn data, before rounding).
        assert w.qblk == BLOCK and w.q_pos0 == 0
        for b in range(w.B):
            for g in range(w.Hkv):
                for i in range(2, w.n_rows):
                    t0, t1 = i * BLOCK, min((i + 1) * BLOCK, w.Tq)
                    qsum = Q[b, t0:t1, g * G:(g + 1) * G, :].sum(dim=(0, 1)).to("cpu")
                    qhat = qsum / qsum.norm()
                    n = min(2, i - 1)
                    js = (torch.randperm(i - 1, generator=pgen)[:n] + 1).tolist()
                    for j in js:
                        adds_k.append((b, g, j, w.plant_scale * qhat))
                        planted.append((b, g, j, i))
    elif w.plant == "partner":
        # A fraction of the cache's complete key blocks (excluding the sink
        # and the last block) per group get a unit direction u added to all
        # 64 keys; u is also added to every query of one partner query row
        # whose diagonal lies after the block.
        assert w.qblk == BLOCK and w.q_pos0 % BLOCK == 0
        first_diag = w.q_pos0 // BLOCK
        if first_diag > 0:      # chunked prefill: plant inside the cache only
            last_cand = first_diag - 1
        else:
            last_cand = min(NB_kv - 2, w.n_rows - 2)
        n_plant = int(w.plant_frac * NB_kv)
        for b in range(w.B):
            for g in range(w.Hkv):
                js = (torch.randperm(last_cand, generator=pgen)[:n_plant] + 1).tolist()
                for j in js:
                    lo = max(0, j + 1 - first_diag)          # rows whose diagonal > j
                    i = lo + int(torch.randint(w.n_rows - lo, (1,), generator=pgen))
                    u = _unit(pgen, w.d)
                    adds_k.append((b, g, j, w.plant_scale * u))
                    adds_q.append((b, g, i, w.plant_scale * u))
                    planted.append((b, g, j, i))

    elif w.plant == "token":
        # Per-token rows (decode): a fraction of the complete key blocks
        # before the first token's diagonal (sink excluded) per group get a
        # unit direction u added to all 64 keys; u is also added to the
        # group's heads of every query token.
        assert w.qblk == 1
        last_cand = w.q_pos0 // BLOCK - 1
        n_plant = int(w.plant_frac * max(last_cand, 0))
        for b in range(w.B):
            for g in range(w.Hkv):
                js = (torch.randperm(last_cand, generator=pgen)[:n_plant] + 1).tolist() if n_plant else []
                for j in js:
                    u = _unit(pgen, w.d)
                    adds_k.append((b, g, j, w.plant_scale * u))
                    for i in range(w.n_rows):
                        adds_q.append((b, g, i, w.plant_scale * u))
                    planted.append((b, g, j, -1))

    for (b, g, i, vec) in adds_q:
        t0, t1 = i * w.qblk, min((i + 1) * w.qblk, w.Tq)
        Q[b, t0:t1, g * G:(g + 1) * G, :] += vec.to(dev)
    Qb = Q.to(torch.bfloat16)
    del Q

    if kv_f32 is not None:
        Kf, Vf = kv_f32
        for (b, g, j, vec) in adds_k:
            Kf[b, g, j * BLOCK:(j + 1) * BLOCK, :] += vec.to(dev)
        K = Kf.to(torch.bfloat16)
        V = Vf.to(torch.bfloat16)
        del Kf, Vf
    else:
        by_b = {}
        for (b, g, j, vec) in adds_k:
            by_b.setdefault(b, []).append((g, j, vec))
        for b in range(w.B):
            kb = torch.randn((w.Hkv, w.T_kv, w.d), generator=gen, device=dev, dtype=torch.float32)
            for (g, j, vec) in by_b.get(b, []):
                kb[g, j * BLOCK:(j + 1) * BLOCK, :] += vec.to(dev)
            K[b].copy_(kb.to(torch.bfloat16))
            del kb
            vb = torch.randn((w.Hkv, w.T_kv, w.d), generator=gen, device=dev, dtype=torch.float32)
            V[b].copy_(vb.to(torch.bfloat16))
            del vb
    return {"Q": Qb, "K": K, "V": V, "planted": planted}


def paged_decode(B=32, min_len=65536, max_len=262144, Hq=16, Hkv=2, d=128, seed=1007,
                 device="cpu"):
    """A ragged decode batch over a paged cache (serving): B single-token
    queries, sequence lengths drawn uniformly in [min_len, max_len], each
    sequence's 64-token blocks in pages [num_pages, Hkv, 64, d] placed by a
    random permutation (the block table), Q, K, V drawn N(0, 1) and rounded
    to bf16 once.  Returns q [B, Hq, d], K_pages, V_pages, block_table
    [B, max_blocks] int32, seq_lens [B] int32 and max_blocks."""
    dev = torch.device(device)
    cpu = torch.Generator(device="cpu")
    cpu.manual_seed(seed)
    lens = torch.randint(min_len, max_len + 1, (B,), generator=cpu, dtype=torch.int64)
    max_blocks = (max_len + BLOCK - 1) // BLOCK
    num_pages = B * max_blocks
    table = torch.randperm(num_pages, generator=cpu).view(B, max_blocks).to(torch.int32)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed + 1)
    q = torch.randn((B, Hq, d), generator=gen, device=dev).to(torch.bfloat16)
    K_pages = torch.empty((num_pages, Hkv, BLOCK, d), device=dev, dtype=torch.bfloat16)
    V_pages = torch.empty_like(K_pages)
    step = 8192   # pages drawn per chunk (bounds the fp32 staging memory)
    for p0 in range(0, num_pages, step):
        n = min(step, num_pages - p0)
        K_pages[p0:p0 + n] = torch.randn((n, Hkv, BLOCK, d), generator=gen, device=dev).to(torch.bfloat16)
        V_pages[p0:p0 + n] = torch.randn((n, Hkv, BLOCK, d), generator=gen, device=dev).to(torch.bfloat16)
    return dict(q=q, K_pages=K_pages, V_pages=V_pages, block_table=table.to(dev),
                seq_lens=lens.to(torch.int32).to(dev), max_blocks=max_blocks, max_len=int(lens.max()))


def paged_prefill(B=8, Tq=4096, min_pos=65536, max_pos=524288, Hq=16, Hkv=2, d=128, seed=1008,
                  device="cpu"):
    """Chunked prefill of a ragged batch over a paged cache: B requests, each
    with Tq new tokens starting at a position drawn uniformly among the
    multiples of 64 in [min_pos, max_pos]; every sequence's blocks (cache and
    chunk) in pages [num_pages, Hkv, 64, d] placed by a random permutation;
    Q, K, V drawn N(0, 1) and rounded to bf16 once.  Returns Q [B, Tq, Hq, d],
    K_pages, V_pages, block_table [B, max_blocks] int32, q_pos [B] int32 and
    max_blocks."""
    dev = torch.device(device)
    cpu = torch.Generator(device="cpu")
    cpu.manual_seed(seed)
    q_pos = BLOCK * torch.randint(min_pos // BLOCK, max_pos // BLOCK + 1, (B,), generator=cpu)
    max_blocks = (max_pos + Tq + BLOCK - 1) // BLOCK
    num_pages = B * max_blocks
    table = torch.randperm(num_pages, generator=cpu).view(B, max_blocks).to(torch.int32)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed + 1)
    Q = torch.randn((B, Tq, Hq, d), generator=gen, device=dev).to(torch.bfloat16)
    K_pages = torch.empty((num_pages, Hkv, BLOCK, d), device=dev, dtype=torch.bfloat16)
    V_pages = torch.empty_like(K_pages)
    step = 8192
    for p0 in range(0, num_pages, step):
        n = min(step, num_pages - p0)
        K_pages[p0:p0 + n] = torch.randn((n, Hkv, BLOCK, d), generator=gen, device=dev).to(torch.bfloat16)
        V_pages[p0:p0 + n] = torch.randn((n, Hkv, BLOCK, d), generator=gen, device=dev).to(torch.bfloat16)
    return dict(Q=Q, K_pages=K_pages, V_pages=V_pages, block_table=table.to(dev),
                q_pos=q_pos.to(torch.int32).to(dev), max_blocks=max_blocks, max_pos=int(q_pos.max()))
