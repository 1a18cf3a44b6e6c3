"""Device-resident state and argument structs for one decode step.

Builds, from synthetic inputs, everything ``ls_decode_step`` needs: indexer key pool
and page tables, the MLA latent KV pool (HBM) or the pinned host history plus the HBM
hot buffer, block summaries for the coarse-to-fine indexer, output tensors and the
caller-owned workspace.  Only allocation and data placement happen here; every step
of the decode path runs in libls.so.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

from . import binding as B
from . import synthetic as syn


def _round4(x):
    return (int(x) + 3) // 4 * 4


@dataclass
class DecodeWorkload:
    name: str
    batch: int
    k: int
    lens: list
    tensors: dict = field(default_factory=dict)
    args: object = None
    workspace: torch.Tensor | None = None
    hotbuf_init: dict | None = None   # pristine hot-buffer state, restored between steps
    kernels_per_step: int = 0

    def step(self, events=None, stream=None):
        a = self.args
        if events is not None:
            a.events = B.C.cast(events, B.C.c_void_p).value
        else:
            a.events = None
        B.ls_decode_step(a, self.workspace, stream=stream)

    def restore_hotbuf(self):
        """Put the hot-buffer state back to its pre-step contents (outside timed regions)."""
        if self.hotbuf_init is None:
            return
        for key, val in self.hotbuf_init.items():
            self.tensors[key].copy_(val, non_blocking=True)

    @property
    def o(self):
        return self.tensors["o"]

    @property
    def lse(self):
        return self.tensors["lse"]

    @property
    def idx(self):
        return self.tensors["idx"]


# the per-step inputs (the queries, head weights, scales, lengths, page tables) and
# outputs of a step: each set lives in one device buffer, so that a step's traffic with the
# host is one copy each way
STEP_INPUTS = ("i_q", "i_q_scale", "i_w", "i_lens", "i_page_table")  # the indexer's
STEP_INPUTS_ATTN = ("a_q",)  # the attention's queries: needed only after the top-k
STEP_OUTPUTS = ("o", "lse")


def _pack(t: dict, names, dev):
    """Rebind t[name] for each name to a view of one shared device buffer (256-byte aligned
    pieces, contents copied); returns the buffer."""
    names = [n for n in names if t.get(n) is not None]
    offs, o = [], 0
    for n in names:
        offs.append(o)
        o += (t[n].numel() * t[n].element_size() + 255) // 256 * 256
    buf = torch.empty(max(o, 256), dtype=torch.uint8, device=dev)
    for n, off in zip(names, offs):
        nbytes = t[n].numel() * t[n].element_size()
        view = buf[off: off + nbytes].view(t[n].dtype).view(t[n].shape)
        view.copy_(t[n])
        t[n] = view
    return buf


def build(name: str, ind: syn.IndexerInputs, *, k: int, attn: dict, device="cuda", hotbuf: dict | None = None,
          c2f: bool = False, eps_rel: float = 0.0, c2f_keys_on_host: bool = False,
          c2f_stage_blocks: int = 0) -> DecodeWorkload:
    """ind: indexer inputs (CPU or device tensors).  attn: dict(q, kv) for MLA (kv = latent
    pool [NP,64,576] bf16, on device or CPU) or dict(q, k, v) for the fp32 path, plus
    scale.  hotbuf: dict(pos_of_slot, slot_of_pos, recent, host_kv (pinned)) to read the
    history from host memory through a 4,096-slot HBM hot buffer."""
    dev = torch.device(device)
    lens = [int(x) for x in ind.lens.tolist()]
    Bn = len(lens)
    ml = _round4(max(lens))
    t = {}
    for key in ("q", "q_scale", "w", "key_pool", "key_scale", "page_table", "lens"):
        v = getattr(ind, key)
        t["i_" + key] = None if v is None else v.to(dev)
    mla = "kv" in attn or "kv_host" in attn
    t["a_q"] = attn["q"].to(dev)
    heads = t["a_q"].shape[1]
    dv = 512 if mla else attn["v"].shape[-1]
    t["o"] = torch.zeros((Bn, heads, dv), dtype=torch.bfloat16 if mla else torch.float32, device=dev)
    t["lse"] = torch.zeros((Bn, heads), dtype=torch.float32, device=dev)
    t["step_in"] = _pack(t, STEP_INPUTS, dev)
    t["step_in_attn"] = _pack(t, STEP_INPUTS_ATTN, dev)
    t["step_out"] = _pack(t, STEP_OUTPUTS, dev)
    ix = B.index_args(q=t["i_q"], w=t["i_w"], key_pool=t["i_key_pool"], page_table=t["i_page_table"],
                      lens=t["i_lens"], q_scale=t["i_q_scale"], key_scale=t["i_key_scale"], max_len=ml)
    t["idx"] = torch.full((Bn, k), -1, dtype=torch.int32, device=dev)
    t["sel"] = torch.zeros((Bn, k), dtype=torch.float32, device=dev)
    hb = None
    if hotbuf is not None:
        n_slots = hotbuf["pos_of_slot"].shape[1]
        host = hotbuf["host_kv"]
        t["host_kv"] = host
        t["pos_of_slot"] = hotbuf["pos_of_slot"].to(dev)
        t["slot_of_pos"] = hotbuf["slot_of_pos"].to(dev)
        t["recent_score"] = hotbuf["recent"].to(dev)
        t["n_miss"] = torch.zeros((Bn,), dtype=torch.int32, device=dev)
        for key in ("sel_slot", "miss_pos", "miss_slot"):  # the resolve's lists, kept for inspection
            t[key] = torch.full((Bn, k), -1, dtype=torch.int32, device=dev)
        # hot buffer rows: the resident positions' KV, copied from the host history
        hbuf = torch.zeros((Bn, n_slots, 576), dtype=torch.bfloat16)
        pt = ind.page_table.cpu()
        pos_of_slot = hotbuf["pos_of_slot"].cpu()
        for b in range(Bn):
            slots = torch.nonzero(pos_of_slot[b] >= 0).flatten()
            pos = pos_of_slot[b, slots].long()
            hbuf[b, slots] = host[pt[b, pos // 64].long(), pos % 64]
        t["hbuf"] = hbuf.to(dev)
        hb = dict(pos_of_slot=t["pos_of_slot"], recent_score=t["recent_score"], slot_of_pos=t["slot_of_pos"],
                  host_kv=host, hbuf=t["hbuf"], n_miss=t["n_miss"], sel_slot=t["sel_slot"],
                  miss_pos=t["miss_pos"], miss_slot=t["miss_slot"])
        at = B.attn_args(q=t["a_q"], k_rows=t["hbuf"], o=t["o"], lse=t["lse"], scale=attn["scale"],
                         n_slots=n_slots, k=k)
    else:
        if mla:
            t["kv"] = attn["kv"].to(dev)
            at = B.attn_args(q=t["a_q"], k_rows=t["kv"], o=t["o"], lse=t["lse"], scale=attn["scale"],
                             page_table=t["i_page_table"], k=k)
        else:
            t["k_pool"] = attn["k"].to(dev)
            t["v_pool"] = attn["v"].to(dev)
            at = B.attn_args(q=t["a_q"], k_rows=t["k_pool"], v_rows=t["v_pool"], o=t["o"], lse=t["lse"],
                             scale=attn["scale"], page_table=t["i_page_table"], k=k)
    cf = None
    if c2f:
        mb = max(-(-L // 64) for L in lens)
        t["summaries"] = torch.zeros((Bn, mb, 256), dtype=torch.uint8, device=dev)
        t["block_scale"] = torch.zeros((Bn, mb), dtype=torch.float32, device=dev)
        t["survivors"] = torch.zeros((Bn, mb), dtype=torch.int32, device=dev)
        t["n_survivors"] = torch.zeros((Bn,), dtype=torch.int32, device=dev)
        B.ls_build_block_summaries(q=t["i_q"], w=t["i_w"], key_pool=t["i_key_pool"], key_scale=t["i_key_scale"],
                                   q_scale=t["i_q_scale"], page_table=t["i_page_table"], lens=t["i_lens"],
                                   max_len=ml, summaries=t["summaries"], block_scale=t["block_scale"])
        if c2f_keys_on_host:
            # only the summaries stay in HBM: the original keys and scales move to pinned host
            # memory, where the step fetches the blocks it needs
            torch.cuda.synchronize()
            t["i_key_pool"] = ind.key_pool.pin_memory()
            t["i_key_scale"] = ind.key_scale.pin_memory()
            ix = B.index_args(q=t["i_q"], w=t["i_w"], key_pool=t["i_key_pool"], page_table=t["i_page_table"],
                              lens=t["i_lens"], q_scale=t["i_q_scale"], key_scale=t["i_key_scale"], max_len=ml)
        cf = dict(summaries=t["summaries"], block_scale=t["block_scale"], survivors=t["survivors"],
                  n_survivors=t["n_survivors"], eps_rel=eps_rel, keys_on_host=c2f_keys_on_host,
                  stage_blocks=c2f_stage_blocks)
    args = B.decode_step_args(index=ix, k=k, attn=at, c2f=cf, hotbuf=hb, idx=t["idx"], sel_score=t["sel"])
    ws_bytes = B.ls_decode_step_workspace_size(args)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    wl = DecodeWorkload(name=name, batch=Bn, k=k, lens=lens, tensors=t, args=args, workspace=ws)
    if hotbuf is not None:
        wl.hotbuf_init = {key: t[key].clone() for key in ("pos_of_slot", "slot_of_pos", "recent_score", "hbuf")}
    wl.kernels_per_step = kernels_per_step(wl, c2f=c2f, hotbuf=hotbuf is not None, mla=mla)
    if c2f and c2f_keys_on_host:
        # a fetch before the candidate blocks' scoring; the survivors' single scoring launch
        # becomes fetch + scoring per staging pass
        mb = t["summaries"].shape[1]
        nb0 = min(mb, (k + 63) // 64 + 1)
        cap = min(mb, max(nb0, c2f_stage_blocks if c2f_stage_blocks > 0 else 2048))
        wl.kernels_per_step += 1 + 2 * (-(-mb // cap)) - 1
    return wl


def kernels_per_step(wl: DecodeWorkload, *, c2f: bool, hotbuf: bool, mla: bool) -> int:
    """How many of the library's kernels one ls_decode_step launches."""
    # indexer + top-k; coarse-to-fine: bound, top-k, phase 1, rescore, top-k, survivors, rescore, top-k
    n = 8 if c2f else 2
    if mla and hotbuf:
        # classify, resolve, gather into staging, staged rows into slots; resident-row
        # pass, miss pass, merge of both passes
        n += 4 + 3
    elif hotbuf:
        n += 2 + 1   # resolve, gather; attention
    elif mla:
        n += 2 if B.ls_sparse_attn_workspace_size(wl.args.attn) > 0 else 1
    else:
        n += 1
    return n


# ----------------------------------------------------------------------------- named configs
def mla_decode(batch=8, ctx=131072, k=2048, seed=1002, device="cuda", kv_on_device=True) -> DecodeWorkload:
    """Batch of requests at one context length; fp8 indexer (64 heads x 128), MLA bf16
    attention (128 heads x 576, V = first 512 dims), paged 64-token caches with shuffled
    page tables, all in HBM."""
    lens = [ctx] * batch
    ind = syn.indexer_fp8(lens, seed=seed)
    n_pool = ind.key_pool.shape[0]
    q, kv = syn.mla_attention(batch, n_pool, seed=seed + 1000, device=device if kv_on_device else "cpu")
    return build(f"mla_decode_b{batch}_ctx{ctx}", ind, k=k, device=device,
                 attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)))


def mla_hotbuf_decode(batch=36, ctx=131072, k=2048, miss_frac=0.2, n_slots=4096, seed=1003,
                      device="cuda", lens=None) -> DecodeWorkload:
    """The hot-buffer configuration: the full KV history in pinned host memory, a
    4,096-slot hot buffer per request in HBM holding all but a seeded ``miss_frac`` of this
    step's selection (the selection of the GPU's own indexer and top-k), filled up with
    other positions.  Restore the buffer state (``restore_hotbuf``) before every step.
    ``lens`` (one length per request) replaces batch x ctx, e.g. a ragged batch."""
    lens = [ctx] * batch if lens is None else [int(x) for x in lens]
    batch, ctx = len(lens), max(lens)
    ind = syn.indexer_fp8(lens, seed=seed)
    n_pool = ind.key_pool.shape[0]
    q, kv_dev = syn.mla_attention(batch, n_pool, seed=seed + 1000, device=device)
    host = torch.empty(kv_dev.shape, dtype=torch.bfloat16, pin_memory=True)
    host.copy_(kv_dev)
    del kv_dev
    ml = _round4(ctx)
    d = {key: getattr(ind, key).to(device) for key in ("q", "q_scale", "w", "key_pool", "key_scale", "page_table",
                                                      "lens")}
    scores = torch.empty((batch, ml), dtype=torch.float32, device=device)
    idx = torch.empty((batch, k), dtype=torch.int32, device=device)
    B.ls_index_score(q=d["q"], w=d["w"], key_pool=d["key_pool"], page_table=d["page_table"], lens=d["lens"],
                     scores=scores, q_scale=d["q_scale"], key_scale=d["key_scale"])
    B.ls_topk_select(scores=scores, lens=d["lens"], idx=idx)
    sel = idx.cpu()
    del d, scores
    pos_of_slot, slot_of_pos, recent = syn.hot_buffer_state([r[r >= 0] for r in sel], lens, n_slots=n_slots,
                                                            miss_frac=miss_frac, seed=seed + 2000, max_len=ml)
    name = f"mla_hotbuf_b{batch}_ctx{ctx}" if len(set(lens)) == 1 else f"mla_hotbuf_ragged_b{batch}"
    return build(f"{name}_miss{int(round(miss_frac * 100))}", ind, k=k, device=device,
                 attn=dict(q=q, kv_host=True, scale=syn.softmax_scale(576)),
                 hotbuf=dict(pos_of_slot=pos_of_slot, slot_of_pos=slot_of_pos, recent=recent, host_kv=host))


def c2f_decode(batch=4, ctx=1048576, k=2048, keys_on_host=False, stage_blocks=0, seed=1004,
               device="cuda") -> DecodeWorkload:
    """The coarse-to-fine configuration: block-clustered fp8 keys (2% of the blocks shifted
    toward the query) at ``ctx`` tokens per request, per-block summaries in HBM, the
    original keys in HBM or (``keys_on_host``) in pinned host memory; MLA attention over a
    paged bf16 pool in HBM."""
    lens = [ctx] * batch
    ind = syn.coarse_to_fine_indexer(lens, seed=seed)
    q, kv = syn.mla_attention(batch, ind.key_pool.shape[0], seed=seed + 1000, device=device)
    where = "hostkeys" if keys_on_host else "hbmkeys"
    return build(f"c2f_b{batch}_ctx{ctx}_{where}", ind, k=k, device=device, c2f=True,
                 attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)), c2f_keys_on_host=keys_on_host,
                 c2f_stage_blocks=stage_blocks)


def tiny_f32(device="cuda") -> DecodeWorkload:
    """One request at 8,192 tokens, fp32 throughout: indexer 8 heads x 64, top-256,
    16 query heads against one 128-dim K head and one 128-dim V head."""
    ind = syn.indexer_f32([8192], heads=8, dim=64, seed=1001)
    q, K, V = syn.f32_attention(1, 128, heads=16, d=128, seed=2001)
    return build("tiny_f32_ctx8192", ind, k=256, device=device, attn=dict(q=q, k=K, v=V, scale=1 / math.sqrt(128)))
