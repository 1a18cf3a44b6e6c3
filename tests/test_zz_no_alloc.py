"""The allocation-free attention entry point gives the same result as the regular one.

ls_sparse_attn_decode_noalloc is for callers that cannot allocate device memory (for
instance code running under another engine's memory manager, which has already
claimed the free HBM, or a C caller without a device allocator): it keeps the split-KV
partials in scratch compiled into the library instead of a caller workspace.  Both entry
points run the same kernels on the same inputs, so their outputs must be identical bit for
bit.  This file is collected last on purpose, so a run that stops at its first failure has
already run every other test; it also passes when run alone in a fresh process.
"""
import math

import pytest
import torch

from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

DEV = "cuda"


BATCH = 10  # seven KV splits per request: their partials go through the split scratch


def _inputs(seed):
    lens = [131072] * BATCH
    table, n_pool = syn.page_layout(lens, seed=seed)
    q, kv = syn.mla_attention(len(lens), n_pool, seed=seed + 1, device=DEV)
    g = torch.Generator().manual_seed(seed + 2)
    sel = torch.stack([torch.randperm(L, generator=g)[:2048].sort().values for L in lens]).to(torch.int32)
    sel[3, 1500:] = -1  # a request with fewer valid rows
    return table.to(DEV), q, kv, sel.to(DEV)


def _run(table, q, kv, sel, noalloc):
    o = torch.full((BATCH, 128, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((BATCH, 128), float("nan"), device=DEV)
    a = B.attn_args(q=q, k_rows=kv, sel=sel, o=o, lse=lse, scale=syn.softmax_scale(576), page_table=table)
    need = B.ls_sparse_attn_workspace_size(a)
    assert need > 0, "this configuration should use split-KV scratch"
    if noalloc:
        B.ls_sparse_attn_decode_noalloc(a)
    else:
        ws = torch.empty(need, dtype=torch.uint8, device=DEV)
        B.ls_sparse_attn_decode(a, ws)
    torch.cuda.synchronize()
    return o, lse


def test_noalloc_attention_matches_workspace_attention_twice():
    for seed in (71, 72):  # two calls in a row share (and overwrite) the built-in scratch
        table, q, kv, sel = _inputs(seed)
        ref_o, ref_lse = _run(table, q, kv, sel, noalloc=False)
        o, lse = _run(table, q, kv, sel, noalloc=True)
        assert torch.isfinite(o.float()).all() and not torch.isnan(lse).any()
        assert torch.equal(o, ref_o)
        assert torch.equal(lse, ref_lse)
    assert B.ls_check_device_status() == 0


def test_noalloc_attention_without_split_scratch():
    """A configuration that needs no split-KV scratch (the fp32 CUDA-core attention): the
    entry point leaves the built-in array alone and returns what the regular call does."""
    q, K, V = syn.f32_attention(1, 128, heads=16, d=128, seed=2001)
    table = torch.arange(128, dtype=torch.int32).view(1, 128)
    sel = torch.arange(0, 8192, 32, dtype=torch.int32).view(1, 256)
    outs = []
    for noalloc in (False, True, True):
        o = torch.full((1, 16, 128), float("nan"), device=DEV)
        lse = torch.full((1, 16), float("nan"), device=DEV)
        a = B.attn_args(q=q.to(DEV), k_rows=K.to(DEV), v_rows=V.to(DEV), sel=sel.to(DEV), o=o, lse=lse,
                        scale=1 / math.sqrt(128), page_table=table.to(DEV))
        assert B.ls_sparse_attn_workspace_size(a) == 0
        if noalloc:
            B.ls_sparse_attn_decode_noalloc(a)
        else:
            B.ls_sparse_attn_decode(a, None)
        torch.cuda.synchronize()
        outs.append((o, lse))
    for o, lse in outs[1:]:
        assert torch.isfinite(o).all()
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])
    assert B.ls_check_device_status() == 0
