"""Context-parallel decode of long requests over G GPUs (one process per GPU).

GPU g holds a contiguous, page-aligned shard of every request's context (its own page
tables into its own pools) and per step: scores and selects over its shard (candidates
with global positions), all-gathers the candidates, takes the global top-k of them (the
same on every GPU, and the same as one GPU scanning the whole context), attends to the
selected rows of its shard, all-gathers the normalised partial outputs with their
log-sum-exp, and merges them.  Every step of the arithmetic runs in the library's
kernels (include/ls.h: ls_index_score, ls_topk_select with pos_offset,
ls_cp_merge_topk, ls_sparse_attn_decode with o_f32, ls_attn_merge); the two exchanges
are NCCL all-gathers through torch.distributed.

The step is split in three phases so that a caller without G GPUs can run the shards
one after another on one GPU and stack their outputs in place of the all-gathers.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as B

PAGE = 64


def shard_ranges(lens, world: int):
    """Page-aligned contiguous shards: (begin, end) per request and rank, covering
    [0, L_b) with page counts differing by at most one between ranks."""
    if world < 1:
        raise ValueError("world must be >= 1")
    out = []
    for L in lens:
        L = int(L)
        pages = -(-L // PAGE)
        base, extra = divmod(pages, world)
        row, p0 = [], 0
        for r in range(world):
            p1 = p0 + base + (1 if r < extra else 0)
            row.append((min(L, p0 * PAGE), min(L, p1 * PAGE)))
            p0 = p1
        out.append(row)
    return out  # [B][world] of (begin, end)


def all_gather(local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """[world, *local.shape], rank order (the local tensor itself for one rank)."""
    if world == 1:
        return local.unsqueeze(0)
    local = local.contiguous()
    out = torch.empty((world * local.shape[0], *local.shape[1:]), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(out, local, group=group)  # ranks concatenated along dim 0
    return out.view(world, *local.shape)


class ShardStep:
    """One GPU's part of a context-parallel decode step.

    index: ls_index_score arguments over this shard (local positions, local lens, local
    page table into this GPU's key pool); attn: dict(q [B,128,576] bf16, kv pool,
    page_table (local), scale); begin / end: [B] int32 CUDA tensors, this shard's global
    range per request."""

    def __init__(self, *, index: B.IndexScoreArgs, k: int, attn: dict, begin: torch.Tensor, end: torch.Tensor,
                 world: int):
        dev = begin.device
        self.index, self.k, self.world = index, k, world
        Bn = index.batch
        self.begin, self.end = begin, end
        self.lens = (end - begin).to(torch.int32)
        self.scores = torch.empty((Bn, index.max_len), dtype=torch.float32, device=dev)
        index.scores = self.scores.data_ptr()
        self.cand_pos = torch.empty((Bn, k), dtype=torch.int32, device=dev)
        self.cand_score = torch.empty((Bn, k), dtype=torch.float32, device=dev)
        self.idx = torch.empty((Bn, k), dtype=torch.int32, device=dev)
        self.sel_score = torch.empty((Bn, k), dtype=torch.float32, device=dev)
        self.local_sel = torch.empty((Bn, k), dtype=torch.int32, device=dev)
        heads, dv = attn["q"].shape[1], 512
        self.o_part = torch.empty((Bn, heads, dv), dtype=torch.float32, device=dev)
        self.lse_part = torch.empty((Bn, heads), dtype=torch.float32, device=dev)
        self.attn = B.attn_args(q=attn["q"], k_rows=attn["kv"], sel=self.local_sel, o=self.o_part, lse=self.lse_part,
                                scale=attn["scale"], page_table=attn["page_table"], k=k)
        self.attn_ws = torch.empty(max(256, B.ls_sparse_attn_workspace_size(self.attn)), dtype=torch.uint8,
                                   device=dev)
        self.merge_ws = None
        self._refs = (attn,)

    def candidates(self):
        """Phase 1: this shard's top-k candidates, global positions and their scores."""
        _check_call(B.lib().ls_index_score(B.C.byref(self.index), B._stream(None)))
        B.ls_topk_select(scores=self.scores, lens=self.lens, idx=self.cand_pos, sel_score=self.cand_score,
                         pos_offset=self.begin)
        return self.cand_score, self.cand_pos

    def attend(self, cand_score_all: torch.Tensor, cand_pos_all: torch.Tensor):
        """Phase 2: the global top-k of the gathered candidates [G,B,k], then attention over
        its rows in this shard; returns the normalised partial (o, lse)."""
        m = B.cp_merge_args(cand_score=cand_score_all, cand_pos=cand_pos_all, shard_begin=self.begin,
                            shard_end=self.end, idx=self.idx, sel_score=self.sel_score, local_sel=self.local_sel)
        need = B.ls_cp_merge_workspace_size(m)
        if self.merge_ws is None or self.merge_ws.numel() < need:
            self.merge_ws = torch.empty(need, dtype=torch.uint8, device=self.begin.device)
        B.ls_cp_merge_topk(m, self.merge_ws)
        B.ls_sparse_attn_decode(self.attn, self.attn_ws)
        return self.o_part, self.lse_part

    def step(self, o: torch.Tensor, lse: torch.Tensor, group=None):
        """The whole step on `world` ranks; o [B,128,512] (bf16 or f32) and lse [B,128] out."""
        cs, cp = self.candidates()
        op, lp = self.attend(all_gather(cs, self.world, group), all_gather(cp, self.world, group))
        B.ls_attn_merge(o_parts=all_gather(op, self.world, group), lse_parts=all_gather(lp, self.world, group),
                        o=o, lse=lse)


def _check_call(status):
    if status != B.LS_OK:
        raise B.LsError(status, B.lib().ls_get_error_string().decode())
