"""Context-parallel split of one request over G shards, run shard after shard on one GPU
(the all-gathers become stacks): the global top-k equals one GPU's full scan exactly and
the merged attention matches the oracle on that selection."""
import numpy as np
import pytest
import torch

import oracle.ls_oracle as O
from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import cp
from sparse_attention_decode_ls_b200 import synthetic as syn

from gpu_helpers import DEV, assert_status_clean, bits16, gpu_index_scores, round4

pytestmark = pytest.mark.gpu


def _shard_args(inp, d, q, kv, ranges, g, k):
    """ls_index_score / attention arguments over shard g of every request: the shard's
    slice of each page table, local positions and lengths."""
    Bn = len(ranges)
    begins = [ranges[b][g][0] for b in range(Bn)]
    ends = [ranges[b][g][1] for b in range(Bn)]
    pages = [-(-(e - s) // 64) for s, e in zip(begins, ends)]
    mp = max(1, max(pages))
    table = torch.zeros((Bn, mp), dtype=torch.int32)
    for b in range(Bn):
        table[b, :pages[b]] = inp.page_table[b, begins[b] // 64: begins[b] // 64 + pages[b]]
    table = table.to(DEV)
    lens = torch.tensor([e - s for s, e in zip(begins, ends)], dtype=torch.int32, device=DEV)
    ml = round4(max(1, int(lens.max())))
    ix = B.index_args(q=d["q"], w=d["w"], key_pool=d["key_pool"], page_table=table, lens=lens, q_scale=d["q_scale"],
                      key_scale=d["key_scale"], max_len=ml)
    attn = dict(q=q, kv=kv, page_table=table, scale=syn.softmax_scale(576))
    return cp.ShardStep(index=ix, k=k, attn=attn, begin=torch.tensor(begins, dtype=torch.int32, device=DEV),
                        end=torch.tensor(ends, dtype=torch.int32, device=DEV), world=len(ranges[0]))


@pytest.mark.parametrize("lens,G", [([64 * 900 + 13, 64 * 700], 3), ([64 * 40 + 5, 3000], 4), ([64 * 500], 1)])
def test_context_parallel_matches_full_scan(lens, G):
    k = 2048
    inp = syn.indexer_fp8(lens, seed=81)
    d = {kk: v.to(DEV) for kk, v in inp.__dict__.items() if isinstance(v, torch.Tensor)}
    q, kv = syn.mla_attention(len(lens), inp.key_pool.shape[0], seed=82)
    qd, kvd = q.to(DEV), kv.to(DEV)
    # one GPU over the whole context
    scores = gpu_index_scores(inp)
    full = torch.empty((len(lens), k), dtype=torch.int32, device=DEV)
    B.ls_topk_select(scores=scores, lens=d["lens"], idx=full)
    # G shards, one after another
    ranges = cp.shard_ranges(lens, G)
    shards = [_shard_args(inp, d, qd, kvd, ranges, g, k) for g in range(G)]
    cands = [s.candidates() for s in shards]
    cs = torch.stack([c[0] for c in cands])
    cpos = torch.stack([c[1] for c in cands])
    parts = [s.attend(cs, cpos) for s in shards]
    o = torch.empty((len(lens), 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((len(lens), 128), device=DEV)
    B.ls_attn_merge(o_parts=torch.stack([p[0] for p in parts]), lse_parts=torch.stack([p[1] for p in parts]),
                    o=o, lse=lse)
    torch.cuda.synchronize()
    assert_status_clean()
    for s in shards:
        assert torch.equal(s.idx, full), "every shard takes the full scan's top-k"
    # the oracle's attention over that selection
    qb, kvb = bits16(q), bits16(kv)
    pt = inp.page_table.numpy()
    for b in range(len(lens)):
        sel = full[b].cpu().numpy()
        rows = O.bf16_decode(O.selected_rows(kvb, pt[b], sel))
        ro, rl = O.sparse_attn_decode(O.bf16_decode(qb[b]), rows, rows[:, :512], syn.softmax_scale(576))
        assert np.abs(o[b].float().cpu().numpy() - ro).max() <= 2e-2
        assert np.abs(lse[b].cpu().numpy() - rl).max() <= 2e-2


def test_attn_merge_of_a_split_selection():
    """Two disjoint halves of one selection, attended separately with float32 partials and
    merged, against the oracle on the whole selection."""
    lens = [64 * 300]
    inp = syn.indexer_fp8(lens, seed=83)
    q, kv = syn.mla_attention(1, inp.key_pool.shape[0], seed=84)
    qd, kvd, pt = q.to(DEV), kv.to(DEV), inp.page_table.to(DEV)
    g = torch.Generator().manual_seed(85)
    sel = torch.randperm(lens[0], generator=g)[:2048].sort().values.to(torch.int32)
    halves = [torch.where(torch.arange(2048) % 2 == h, sel, torch.full_like(sel, -1))[None].to(DEV) for h in (0, 1)]
    ops, lps = [], []
    for hsel in halves:
        op = torch.empty((1, 128, 512), device=DEV)
        lp = torch.empty((1, 128), device=DEV)
        a = B.attn_args(q=qd, k_rows=kvd, sel=hsel, o=op, lse=lp, scale=syn.softmax_scale(576), page_table=pt)
        B.ls_sparse_attn_decode(a, torch.empty(max(256, B.ls_sparse_attn_workspace_size(a)), dtype=torch.uint8,
                                               device=DEV))
        ops.append(op)
        lps.append(lp)
    o = torch.empty((1, 128, 512), device=DEV)
    lse = torch.empty((1, 128), device=DEV)
    B.ls_attn_merge(o_parts=torch.stack(ops), lse_parts=torch.stack(lps), o=o, lse=lse)
    torch.cuda.synchronize()
    assert_status_clean()
    rows = O.bf16_decode(O.selected_rows(bits16(kv), inp.page_table.numpy()[0], sel.numpy()))
    ro, rl = O.sparse_attn_decode(O.bf16_decode(bits16(q)[0]), rows, rows[:, :512], syn.softmax_scale(576))
    assert np.abs(o[0].cpu().numpy() - ro).max() <= 5e-3  # float32 partials and output (P is bf16)
    assert np.abs(lse[0].cpu().numpy() - rl).max() <= 5e-3
