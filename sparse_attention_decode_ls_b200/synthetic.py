"""Seeded synthetic inputs shaped like the workloads the pages describe.

This module only draws random numbers and lays them out (fp8 quantisation of the
drawn values included: the path consumes fp8 inputs).  It holds none of the decode
path's arithmetic and imports neither the CUDA binding nor the oracle; tests and
the benchmark feed the same tensors to both.

Every generator returns CPU tensors unless ``device`` says otherwise.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

PAGE = 64
FP8_MAX = 448.0


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def quantize_e4m3(x: torch.Tensor, dim: int = -1):
    """Per-row e4m3 quantisation with scale amax/448 (the recipe for the indexer's
    fp8 keys and query).  Returns (uint8 codes, float32 scales)."""
    amax = x.abs().amax(dim=dim, keepdim=True).clamp_min(1e-12)
    scale = (amax / FP8_MAX).float()
    codes = (x / scale).clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.squeeze(dim).contiguous()


def page_layout(lens, seed: int, max_pages: int | None = None):
    """A pool of exactly sum(ceil(L_b/64)) pages, handed out to the requests through a
    seeded random permutation (shuffled page tables).  Unused table entries are 0."""
    lens = [int(x) for x in lens]
    n_pages = [-(-L // PAGE) for L in lens]
    total = sum(n_pages)
    if max_pages is None:
        max_pages = max(max(n_pages), 1)
    perm = torch.randperm(total, generator=_gen(seed))
    table = torch.zeros((len(lens), max_pages), dtype=torch.int32)
    off = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[off: off + n].to(torch.int32)
        off += n
    return table, total


@dataclass
class IndexerInputs:
    lens: torch.Tensor            # [B] int32
    page_table: torch.Tensor      # [B, maxP] int32
    q: torch.Tensor               # [B,H,D] uint8 e4m3 codes, or float32
    q_scale: torch.Tensor | None  # [B,H] float32
    w: torch.Tensor               # [B,H] bfloat16 or float32
    key_pool: torch.Tensor        # [NP,64,D] uint8 codes, or float32
    key_scale: torch.Tensor | None  # [NP,64] float32
    key_format: str = "e4m3"
    extra: dict = field(default_factory=dict)

    @property
    def batch(self):
        return int(self.lens.shape[0])

    @property
    def max_len(self):
        return int(self.lens.max())


def indexer_fp8(lens, *, heads=64, dim=128, seed=1002, w_std=0.1, w_nonneg=False,
                keys: torch.Tensor | None = None, q: torch.Tensor | None = None,
                max_pages=None) -> IndexerInputs:
    """fp8 indexer inputs: q ~ N(0,1) quantised per head, keys ~ N(0,1) (or the given
    float keys, one row per pool token) quantised per token, w ~ N(0, w_std) in bf16
    (absolute value when ``w_nonneg``), shuffled 64-token pages."""
    lens = [int(x) for x in lens]
    B = len(lens)
    g = _gen(seed)
    table, n_pool = page_layout(lens, seed + 17, max_pages)
    if q is None:
        q = torch.randn((B, heads, dim), generator=g)
    q8, sq = quantize_e4m3(q)
    w = torch.randn((B, heads), generator=g) * w_std
    if w_nonneg:
        w = w.abs()
    w = w.to(torch.bfloat16)
    if keys is None:
        keys = torch.randn((n_pool * PAGE, dim), generator=g)
    k8, sk = quantize_e4m3(keys)
    return IndexerInputs(
        lens=torch.tensor(lens, dtype=torch.int32), page_table=table, q=q8, q_scale=sq, w=w,
        key_pool=k8.view(n_pool, PAGE, dim), key_scale=sk.view(n_pool, PAGE), key_format="e4m3")


def indexer_f32(lens, *, heads=8, dim=64, seed=1001) -> IndexerInputs:
    """fp32 indexer inputs: q, k ~ N(0,1), w ~ U(0,1); identity page table."""
    lens = [int(x) for x in lens]
    B = len(lens)
    g = _gen(seed)
    n_pages = [-(-L // PAGE) for L in lens]
    n_pool = sum(n_pages)
    table = torch.zeros((B, max(n_pages)), dtype=torch.int32)
    off = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = torch.arange(off, off + n, dtype=torch.int32)
        off += n
    q = torch.randn((B, heads, dim), generator=g)
    w = torch.rand((B, heads), generator=g)
    keys = torch.randn((n_pool, PAGE, dim), generator=g)
    return IndexerInputs(lens=torch.tensor(lens, dtype=torch.int32), page_table=table, q=q,
                         q_scale=None, w=w, key_pool=keys, key_scale=None, key_format="f32")


def clustered_keys(n_blocks_per_req, B, *, dim=128, within_sigma=0.05, shift_frac=0.02,
                   shift=1.5, direction: torch.Tensor | None = None, seed=1004):
    """Block-clustered float keys: each 64-token block has a centroid c_j ~ N(0, I) and
    its tokens are c_j + within_sigma * N(0, I); a seeded ``shift_frac`` of the blocks
    get c_j += shift * sign(direction[b]) (shifted toward the query).  Returns
    [B * n_blocks * 64, dim] float32 in request-major logical order."""
    g = _gen(seed)
    out = []
    for b in range(B):
        c = torch.randn((n_blocks_per_req, dim), generator=g)
        n_shift = int(round(shift_frac * n_blocks_per_req))
        if n_shift and direction is not None:
            pick = torch.randperm(n_blocks_per_req, generator=g)[:n_shift]
            c[pick] += shift * torch.sign(direction[b])[None, :]
        tok = c[:, None, :] + within_sigma * torch.randn((n_blocks_per_req, PAGE, dim), generator=g)
        out.append(tok.reshape(-1, dim))
    return torch.cat(out, 0)


def coarse_to_fine_indexer(lens, *, seed=1004, sigma=0.05, shift_frac=0.02) -> IndexerInputs:
    """fp8 indexer inputs with block-clustered keys (see ``clustered_keys``): q ~ N(0,1),
    w = |N(0, 0.1)|, and the shifted blocks moved toward sum_h w_h q_h of their request."""
    lens = [int(x) for x in lens]
    B = len(lens)
    g = _gen(seed)
    qf = torch.randn((B, 64, 128), generator=g)
    table, n_pool = page_layout(lens, seed + 17)
    w = (torch.randn((B, 64), generator=g) * 0.1).abs()
    direction = (w[:, :, None] * qf).sum(1)
    keys = torch.cat([clustered_keys(-(-L // PAGE), 1, within_sigma=sigma, shift_frac=shift_frac,
                                     direction=direction[b:b + 1], seed=seed + 1 + b)[:L]
                      for b, L in enumerate(lens)])
    pool_keys = logical_to_pool(keys, lens, table, n_pool)
    del keys
    return indexer_fp8(lens, seed=seed, w_nonneg=True, q=qf, keys=pool_keys)


def logical_to_pool(keys_logical: torch.Tensor, lens, page_table: torch.Tensor, n_pool: int):
    """Place per-request logical token rows into pool rows through the page table."""
    dim = keys_logical.shape[-1]
    pool = torch.zeros((n_pool, PAGE, dim), dtype=keys_logical.dtype)
    off = 0
    for b, L in enumerate(lens):
        n = -(-int(L) // PAGE)
        rows = torch.zeros((n * PAGE, dim), dtype=keys_logical.dtype)
        rows[:L] = keys_logical[off: off + L]
        pool[page_table[b, :n].long()] = rows.view(n, PAGE, dim)
        off += int(L)
    return pool.reshape(n_pool * PAGE, dim)


def mla_attention(batch, n_pool_pages, *, heads=128, dk=576, seed=2002, device="cpu"):
    """MLA-absorbed attention inputs: q ~ N(0,1) bf16 [B, heads, dk]; the latent KV pool
    ~ N(0,1) bf16 [n_pool_pages, 64, dk] (its first 512 dims serve as V)."""
    if device == "cpu":
        g = _gen(seed)
        q = torch.randn((batch, heads, dk), generator=g).to(torch.bfloat16)
        kv = torch.randn((n_pool_pages, PAGE, dk), generator=g).to(torch.bfloat16)
    else:
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        q = torch.randn((batch, heads, dk), generator=g, device=device).to(torch.bfloat16)
        kv = torch.empty((n_pool_pages, PAGE, dk), dtype=torch.bfloat16, device=device)
        chunk = 1024
        for i in range(0, n_pool_pages, chunk):
            j = min(n_pool_pages, i + chunk)
            kv[i:j] = torch.randn((j - i, PAGE, dk), generator=g, device=device).to(torch.bfloat16)
    return q, kv


def f32_attention(batch, n_pool_pages, *, heads=16, d=128, seed=2001):
    """fp32 attention inputs with separate K and V pools: q, K, V ~ N(0,1)."""
    g = _gen(seed)
    q = torch.randn((batch, heads, d), generator=g)
    k = torch.randn((n_pool_pages, PAGE, d), generator=g)
    v = torch.randn((n_pool_pages, PAGE, d), generator=g)
    return q, k, v


def hot_buffer_state(selected, lens, *, n_slots=4096, miss_frac=0.2, seed=3003, max_len=None):
    """Hot-buffer state in which a controlled fraction of a given selection misses.

    ``selected[b]`` lists request b's selected positions.  A seeded random
    round(miss_frac * |S_b|) of them are left out of the buffer (they will miss);
    the rest are resident, and the remaining slots hold seeded random non-selected
    positions, so the buffer is full.  Slots are a random permutation; recent scores
    ~ U(0,1).  Returns (pos_of_slot [B,S] int32, slot_of_pos [B,max_len] int32,
    recent_score [B,S] float32)."""
    B = len(lens)
    max_len = max_len or max(int(x) for x in lens)
    g = _gen(seed)
    pos_of_slot = torch.full((B, n_slots), -1, dtype=torch.int32)
    slot_of_pos = torch.full((B, max_len), -1, dtype=torch.int32)
    recent = torch.rand((B, n_slots), generator=g)
    for b in range(B):
        L = int(lens[b])
        sel = torch.as_tensor(selected[b], dtype=torch.int64)
        sel = sel[sel >= 0]
        n_miss = int(round(miss_frac * sel.numel()))
        perm = torch.randperm(sel.numel(), generator=g)
        resident_sel = sel[perm[n_miss:]]
        is_sel = torch.zeros(L, dtype=torch.bool)
        is_sel[sel] = True
        others = torch.nonzero(~is_sel).flatten()
        others = others[torch.randperm(others.numel(), generator=g)]
        n_fill = min(n_slots - resident_sel.numel(), others.numel())
        resident = torch.cat([resident_sel, others[:n_fill]])
        slots = torch.randperm(n_slots, generator=g)[: resident.numel()]
        pos_of_slot[b, slots] = resident.to(torch.int32)
        slot_of_pos[b, resident] = slots.to(torch.int32)
    return pos_of_slot, slot_of_pos, recent


def ragged_lens(batch, lo=4096, hi=16384, seed=1005):
    """Context lengths ~ U[lo, hi] (integers), seeded."""
    g = _gen(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (batch,), generator=g)]


def softmax_scale(dk: int) -> float:
    return 1.0 / math.sqrt(dk)
