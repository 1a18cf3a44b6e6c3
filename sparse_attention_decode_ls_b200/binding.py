"""ctypes binding of the C ABI in include/ls.h.

Argument marshalling only: every function builds the C argument struct from torch
tensors (shapes and dtypes give the sizes), calls the library and raises LsError on a
non-OK status.  All arithmetic happens in the CUDA kernels of libls.so; there is no
other code path, and a missing library is an error.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libls.so")

LS_OK, LS_ERR_INVALID_ARG, LS_ERR_UNSUPPORTED, LS_ERR_CUDA, LS_ERR_DEVICE_STATUS = range(5)
LS_F32, LS_BF16, LS_E4M3 = 0, 1, 2
LS_ROWS_PAGED, LS_ROWS_SLOTS = 0, 1
LS_DEV_BOUNDS, LS_DEV_TIMEOUT, LS_DEV_CAPACITY = 1, 2, 4

_i32, _i64, _f32, _p = C.c_int32, C.c_int64, C.c_float, C.c_void_p


class IndexScoreArgs(C.Structure):
    _fields_ = [("batch", _i32), ("heads", _i32), ("dim", _i32), ("max_pages", _i32), ("max_len", _i32),
                ("key_dtype", _i32), ("w_dtype", _i32), ("variant", _i32), ("num_pages", _i64),
                ("q", _p), ("q_scale", _p), ("w", _p), ("key_pool", _p), ("key_scale", _p),
                ("page_table", _p), ("lens", _p), ("scores", _p)]


class TopkArgs(C.Structure):
    _fields_ = [("batch", _i32), ("k", _i32), ("max_len", _i32), ("scores", _p), ("lens", _p), ("idx", _p),
                ("sel_score", _p), ("pos_offset", _p)]


class BlockBoundPruneArgs(C.Structure):
    _fields_ = [("index", IndexScoreArgs), ("k", _i32), ("max_blocks", _i32), ("eps_rel", _f32),
                ("summaries", _p), ("block_scale", _p), ("idx", _p), ("sel_score", _p), ("survivors", _p),
                ("n_survivors", _p), ("ub", _p), ("keys_on_host", _i32), ("stage_blocks", _i32)]


class HotbufArgs(C.Structure):
    _fields_ = [("batch", _i32), ("k", _i32), ("n_slots", _i32), ("max_len", _i32), ("sel", _p),
                ("sel_score", _p), ("pos_of_slot", _p), ("recent_score", _p), ("slot_of_pos", _p),
                ("sel_slot", _p), ("miss_pos", _p), ("miss_slot", _p), ("n_miss", _p)]


class GatherArgs(C.Structure):
    _fields_ = [("batch", _i32), ("k", _i32), ("n_slots", _i32), ("max_pages", _i32), ("row_bytes", _i64),
                ("num_pages", _i64), ("host_kv", _p), ("page_table", _p), ("miss_pos", _p), ("miss_slot", _p),
                ("n_miss", _p), ("hbuf", _p)]


class SparseAttnArgs(C.Structure):
    _fields_ = [("batch", _i32), ("heads", _i32), ("dk", _i32), ("dv", _i32), ("k", _i32), ("dtype", _i32),
                ("variant", _i32), ("softmax_scale", _f32), ("addressing", _i32), ("max_pages", _i32),
                ("n_slots", _i32), ("row_stride", _i64), ("num_rows", _i64), ("q", _p), ("k_rows", _p),
                ("v_rows", _p), ("page_table", _p), ("sel", _p), ("o", _p), ("lse", _p), ("o_f32", _i32)]


class CpMergeArgs(C.Structure):
    _fields_ = [("shards", _i32), ("batch", _i32), ("k", _i32), ("cand_score", _p), ("cand_pos", _p),
                ("shard_begin", _p), ("shard_end", _p), ("idx", _p), ("sel_score", _p), ("local_sel", _p)]


class AttnMergeArgs(C.Structure):
    _fields_ = [("parts", _i32), ("batch", _i32), ("heads", _i32), ("dv", _i32), ("o_parts", _p),
                ("lse_parts", _p), ("o", _p), ("o_dtype", _i32), ("lse", _p)]


class DecodeStepArgs(C.Structure):
    _fields_ = [("index", IndexScoreArgs), ("k", _i32), ("use_c2f", _i32), ("max_blocks", _i32),
                ("eps_rel", _f32), ("summaries", _p), ("block_scale", _p), ("survivors", _p),
                ("n_survivors", _p), ("c2f_keys_on_host", _i32), ("c2f_stage_blocks", _i32),
                ("attn", SparseAttnArgs), ("use_hotbuf", _i32), ("n_slots", _i32),
                ("pos_of_slot", _p), ("recent_score", _p), ("slot_of_pos", _p), ("host_kv", _p),
                ("host_num_pages", _i64), ("hbuf", _p), ("n_miss", _p), ("idx", _p), ("sel_score", _p),
                ("events", _p), ("attn_q_ready", _p), ("sel_slot", _p), ("miss_pos", _p), ("miss_slot", _p)]


class PrefillStreamArgs(C.Structure):
    _fields_ = [("layers", _i32), ("batch", _i32), ("max_pages", _i32), ("max_len", _i32), ("max_blocks", _i32),
                ("n_slots", _i32), ("num_pages", _i64), ("row_bytes", _i64), ("page_table", _p), ("lens", _p),
                ("host_keys", _p), ("host_key_scales", _p), ("summaries", _p), ("block_scale", _p),
                ("host_kv", _p), ("hbuf", _p), ("pos_of_slot", _p), ("slot_of_pos", _p), ("recent_score", _p)]


STRUCTS = {"ls_index_score_args": IndexScoreArgs, "ls_topk_args": TopkArgs,
           "ls_prefill_stream_args": PrefillStreamArgs, "ls_cp_merge_args": CpMergeArgs,
           "ls_attn_merge_args": AttnMergeArgs,
           "ls_block_bound_prune_args": BlockBoundPruneArgs, "ls_hotbuf_args": HotbufArgs,
           "ls_gather_args": GatherArgs, "ls_sparse_attn_args": SparseAttnArgs,
           "ls_decode_step_args": DecodeStepArgs}


class LsError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"ls status {status}: {message}")
        self.status = status


_lib = None


def lib():
    """Load libls.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LsError(LS_ERR_UNSUPPORTED, f"{LIB_PATH} is missing: run "
                          "`python -m sparse_attention_decode_ls_b200.build`")
        L = C.CDLL(LIB_PATH)
        P = C.POINTER
        for name, st in [("ls_index_score", IndexScoreArgs), ("ls_topk_select", TopkArgs),
                         ("ls_hotbuf_resolve", HotbufArgs), ("ls_gather_misses", GatherArgs)]:
            f = getattr(L, name)
            f.argtypes = [P(st), _p]
            f.restype = C.c_int
        for name, st in [("ls_sparse_attn_decode", SparseAttnArgs), ("ls_block_bound_prune", BlockBoundPruneArgs),
                         ("ls_decode_step", DecodeStepArgs)]:
            f = getattr(L, name)
            f.argtypes = [P(st), _p, C.c_size_t, _p]
            f.restype = C.c_int
        for name, st in [("ls_sparse_attn_workspace_size", SparseAttnArgs),
                         ("ls_block_bound_prune_workspace_size", BlockBoundPruneArgs),
                         ("ls_decode_step_workspace_size", DecodeStepArgs)]:
            f = getattr(L, name)
            f.argtypes = [P(st)]
            f.restype = C.c_size_t
        L.ls_cp_merge_workspace_size.argtypes = [P(CpMergeArgs)]
        L.ls_cp_merge_workspace_size.restype = C.c_size_t
        L.ls_cp_merge_topk.argtypes = [P(CpMergeArgs), _p, C.c_size_t, _p]
        L.ls_cp_merge_topk.restype = C.c_int
        L.ls_attn_merge.argtypes = [P(AttnMergeArgs), _p]
        L.ls_attn_merge.restype = C.c_int
        L.ls_prefill_stream_workspace_size.argtypes = [P(PrefillStreamArgs)]
        L.ls_prefill_stream_workspace_size.restype = C.c_size_t
        L.ls_prefill_stream.argtypes = [P(PrefillStreamArgs), _p, C.c_size_t, _p]
        L.ls_prefill_stream.restype = C.c_int
        L.ls_sparse_attn_decode_noalloc.argtypes = [P(SparseAttnArgs), _p]
        L.ls_sparse_attn_decode_noalloc.restype = C.c_int
        L.ls_build_block_summaries.argtypes = [P(IndexScoreArgs), _p, _p, _i32, _p]
        L.ls_build_block_summaries.restype = C.c_int
        L.ls_set_wait_limit.argtypes = [C.c_uint64]
        L.ls_set_wait_limit.restype = C.c_int
        L.ls_selftest_bounded_wait.argtypes = [_p]
        L.ls_selftest_bounded_wait.restype = C.c_int
        L.ls_get_error_string.restype = C.c_char_p
        L.ls_version.restype = C.c_char_p
        L.ls_check_device_status.argtypes = [_p, P(C.c_uint32)]
        L.ls_check_device_status.restype = C.c_int
        _lib = L
    return _lib


def _check(status):
    if status != LS_OK:
        raise LsError(status, lib().ls_get_error_string().decode())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _hold(a, *objs):
    """Keep the tensors whose addresses an argument struct holds alive for as long as the
    struct: without this, a temporary such as ``x.to("cuda")`` passed to a builder is
    freed on return and its memory handed to the next allocation (often the workspace)
    before the kernel that reads it runs.  Nested structs bring their own references."""
    refs = list(getattr(a, "_refs", ()))
    for o in objs:
        if o is None:
            continue
        if isinstance(o, dict):
            refs.extend(v for v in o.values() if v is not None)
        elif isinstance(o, C.Structure):
            refs.extend(getattr(o, "_refs", ()))
        else:
            refs.append(o)
    a._refs = refs
    return a


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dt(t):
    return {torch.float32: LS_F32, torch.bfloat16: LS_BF16, torch.uint8: LS_E4M3,
            torch.float8_e4m3fn: LS_E4M3}[t.dtype]


def version() -> str:
    return lib().ls_version().decode()


# ------------------------------------------------------------------------------- a1
def index_args(*, q, w, key_pool, page_table, lens, scores=None, q_scale=None, key_scale=None, max_len=None,
               variant=0) -> IndexScoreArgs:
    B, H, D = q.shape
    a = IndexScoreArgs()
    a.batch, a.heads, a.dim = B, H, D
    a.max_pages = page_table.shape[1]
    a.max_len = int(max_len if max_len is not None else scores.shape[1])
    a.key_dtype = _dt(key_pool)
    a.w_dtype = _dt(w)
    a.variant = variant
    a.num_pages = key_pool.shape[0]
    a.q, a.q_scale, a.w = _ptr(q), _ptr(q_scale), _ptr(w)
    a.key_pool, a.key_scale = _ptr(key_pool), _ptr(key_scale)
    a.page_table, a.lens, a.scores = _ptr(page_table), _ptr(lens), _ptr(scores)
    return _hold(a, q, q_scale, w, key_pool, key_scale, page_table, lens, scores)


def ls_index_score(*, q, w, key_pool, page_table, lens, scores, q_scale=None, key_scale=None, variant=0,
                   stream=None):
    a = index_args(q=q, w=w, key_pool=key_pool, page_table=page_table, lens=lens, scores=scores,
                   q_scale=q_scale, key_scale=key_scale, variant=variant)
    _check(lib().ls_index_score(C.byref(a), _stream(stream)))


# ------------------------------------------------------------------------------- a2
def ls_topk_select(*, scores, lens, idx, sel_score=None, pos_offset=None, stream=None):
    a = TopkArgs()
    a.batch, a.k, a.max_len = scores.shape[0], idx.shape[1], scores.shape[1]
    a.scores, a.lens, a.idx, a.sel_score = _ptr(scores), _ptr(lens), _ptr(idx), _ptr(sel_score)
    a.pos_offset = _ptr(pos_offset)
    _check(lib().ls_topk_select(C.byref(a), _stream(stream)))


# ------------------------------------------------------------------------------- a3
def ls_build_block_summaries(*, q, w, key_pool, key_scale, q_scale, page_table, lens, max_len, summaries,
                             block_scale, stream=None):
    a = index_args(q=q, w=w, key_pool=key_pool, page_table=page_table, lens=lens, q_scale=q_scale,
                   key_scale=key_scale, max_len=max_len)
    _check(lib().ls_build_block_summaries(C.byref(a), _ptr(summaries), _ptr(block_scale),
                                          summaries.shape[1], _stream(stream)))


def c2f_args(*, index: IndexScoreArgs, k, summaries, block_scale, idx, sel_score=None, survivors=None,
             n_survivors=None, ub=None, eps_rel=0.0, keys_on_host=False, stage_blocks=0) -> BlockBoundPruneArgs:
    """keys_on_host: index's key_pool / key_scale are pinned CPU tensors (only the summaries
    are on the GPU); stage_blocks: staging capacity per request and pass (0: default)."""
    a = BlockBoundPruneArgs()
    a.keys_on_host = 1 if keys_on_host else 0
    a.stage_blocks = stage_blocks
    a.index = index
    a.k = k
    a.max_blocks = summaries.shape[1]
    a.eps_rel = eps_rel
    a.summaries, a.block_scale = _ptr(summaries), _ptr(block_scale)
    a.idx, a.sel_score, a.survivors = _ptr(idx), _ptr(sel_score), _ptr(survivors)
    a.n_survivors, a.ub = _ptr(n_survivors), _ptr(ub)
    return _hold(a, index, summaries, block_scale, idx, sel_score, survivors, n_survivors, ub)


def ls_block_bound_prune_workspace_size(a: BlockBoundPruneArgs) -> int:
    return lib().ls_block_bound_prune_workspace_size(C.byref(a))


def ls_block_bound_prune(a: BlockBoundPruneArgs, workspace, stream=None):
    _check(lib().ls_block_bound_prune(C.byref(a), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                      _stream(stream)))


# ------------------------------------------------------------------------------- a4, a5
def ls_hotbuf_resolve(*, sel, sel_score, pos_of_slot, recent_score, slot_of_pos, sel_slot, miss_pos, miss_slot,
                      n_miss, stream=None):
    a = HotbufArgs()
    a.batch, a.k = sel.shape
    a.n_slots = pos_of_slot.shape[1]
    a.max_len = slot_of_pos.shape[1]
    a.sel, a.sel_score = _ptr(sel), _ptr(sel_score)
    a.pos_of_slot, a.recent_score, a.slot_of_pos = _ptr(pos_of_slot), _ptr(recent_score), _ptr(slot_of_pos)
    a.sel_slot, a.miss_pos, a.miss_slot, a.n_miss = _ptr(sel_slot), _ptr(miss_pos), _ptr(miss_slot), _ptr(n_miss)
    _check(lib().ls_hotbuf_resolve(C.byref(a), _stream(stream)))


def ls_gather_misses(*, host_kv, page_table, miss_pos, miss_slot, n_miss, hbuf, stream=None):
    """host_kv: pinned CPU tensor [num_pages, 64, row] (its address is device-accessible
    under unified addressing); hbuf: CUDA tensor [B, n_slots, row]."""
    a = GatherArgs()
    a.batch, a.k = miss_pos.shape
    a.n_slots = hbuf.shape[1]
    a.max_pages = page_table.shape[1]
    a.row_bytes = hbuf.shape[2] * hbuf.element_size()
    a.num_pages = host_kv.shape[0]
    a.host_kv, a.page_table = _ptr(host_kv), _ptr(page_table)
    a.miss_pos, a.miss_slot, a.n_miss, a.hbuf = _ptr(miss_pos), _ptr(miss_slot), _ptr(n_miss), _ptr(hbuf)
    _check(lib().ls_gather_misses(C.byref(a), _stream(stream)))


# ------------------------------------------------------------------------------- a6
def attn_args(*, q, k_rows, v_rows=None, sel=None, o, lse, scale, page_table=None, n_slots=0, dv=None,
              variant=0, k=None) -> SparseAttnArgs:
    """k_rows / v_rows: row pools [..., row_width] (paged pool [NP,64,W] or hot buffer [B,S,W])."""
    v_rows = k_rows if v_rows is None else v_rows
    a = SparseAttnArgs()
    a.batch, a.heads, a.dk = q.shape
    a.dv = int(dv if dv is not None else o.shape[2])
    a.k = int(k if k is not None else sel.shape[1])
    a.dtype = _dt(q)
    a.variant = variant
    a.softmax_scale = scale
    a.addressing = LS_ROWS_PAGED if page_table is not None else LS_ROWS_SLOTS
    a.max_pages = 0 if page_table is None else page_table.shape[1]
    a.n_slots = n_slots if page_table is None else 0
    a.row_stride = k_rows.shape[-1]
    a.num_rows = k_rows.numel() // k_rows.shape[-1]
    a.q, a.k_rows, a.v_rows = _ptr(q), _ptr(k_rows), _ptr(v_rows)
    a.page_table, a.sel, a.o, a.lse = _ptr(page_table), _ptr(sel), _ptr(o), _ptr(lse)
    a.o_f32 = 1 if (o.dtype == torch.float32 and q.dtype == torch.bfloat16) else 0
    return _hold(a, q, k_rows, v_rows, page_table, sel, o, lse)


def ls_sparse_attn_workspace_size(a: SparseAttnArgs) -> int:
    return lib().ls_sparse_attn_workspace_size(C.byref(a))


def ls_sparse_attn_decode(a: SparseAttnArgs, workspace=None, stream=None):
    _check(lib().ls_sparse_attn_decode(C.byref(a), _ptr(workspace),
                                       0 if workspace is None else workspace.numel(), _stream(stream)))


def ls_sparse_attn_decode_noalloc(a: SparseAttnArgs, stream=None):
    """Allocation-free attention: the split-KV partials use the library's built-in
    scratch instead of a caller workspace (see include/ls.h)."""
    _check(lib().ls_sparse_attn_decode_noalloc(C.byref(a), _stream(stream)))


# ------------------------------------------------------------------------------- a7
def decode_step_args(*, index: IndexScoreArgs, k, attn: SparseAttnArgs, c2f=None, hotbuf=None, idx=None,
                     sel_score=None, events=None) -> DecodeStepArgs:
    """c2f: dict(summaries, block_scale, survivors=None, n_survivors=None, eps_rel=0.0,
    keys_on_host=False, stage_blocks=0);
    hotbuf: dict(pos_of_slot, recent_score, slot_of_pos, host_kv, hbuf, n_miss=None,
    sel_slot=None, miss_pos=None, miss_slot=None).
    events: optional ctypes array of 6 cudaEvent_t handles."""
    a = DecodeStepArgs()
    a.index = index
    a.k = k
    a.attn = attn
    if c2f is not None:
        a.use_c2f = 1
        a.max_blocks = c2f["summaries"].shape[1]
        a.eps_rel = c2f.get("eps_rel", 0.0)
        a.summaries, a.block_scale = _ptr(c2f["summaries"]), _ptr(c2f["block_scale"])
        a.survivors, a.n_survivors = _ptr(c2f.get("survivors")), _ptr(c2f.get("n_survivors"))
        a.c2f_keys_on_host = 1 if c2f.get("keys_on_host") else 0
        a.c2f_stage_blocks = int(c2f.get("stage_blocks", 0))
    if hotbuf is not None:
        a.use_hotbuf = 1
        a.n_slots = hotbuf["pos_of_slot"].shape[1]
        a.pos_of_slot, a.recent_score = _ptr(hotbuf["pos_of_slot"]), _ptr(hotbuf["recent_score"])
        a.slot_of_pos, a.host_kv = _ptr(hotbuf["slot_of_pos"]), _ptr(hotbuf["host_kv"])
        a.host_num_pages = hotbuf["host_kv"].shape[0]
        a.hbuf, a.n_miss = _ptr(hotbuf["hbuf"]), _ptr(hotbuf.get("n_miss"))
        a.sel_slot, a.miss_pos = _ptr(hotbuf.get("sel_slot")), _ptr(hotbuf.get("miss_pos"))
        a.miss_slot = _ptr(hotbuf.get("miss_slot"))
    a.idx, a.sel_score = _ptr(idx), _ptr(sel_score)
    a.events = None if events is None else C.cast(events, C.c_void_p).value
    return _hold(a, index, attn, c2f, hotbuf, idx, sel_score, events)


def ls_decode_step_workspace_size(a: DecodeStepArgs) -> int:
    return lib().ls_decode_step_workspace_size(C.byref(a))


def ls_decode_step(a: DecodeStepArgs, workspace, stream=None):
    _check(lib().ls_decode_step(C.byref(a), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                _stream(stream)))


def ls_check_device_status(stream=None) -> int:
    """Synchronise, return and clear the device status bits (LS_DEV_*)."""
    flags = C.c_uint32(0)
    st = lib().ls_check_device_status(_stream(stream), C.byref(flags))
    if st not in (LS_OK, LS_ERR_DEVICE_STATUS):
        _check(st)
    return int(flags.value)


def event_array(events):
    """ctypes array of raw cudaEvent_t handles from torch.cuda.Event objects (None:
    that stage boundary is not recorded)."""
    arr = (C.c_void_p * len(events))()
    for i, e in enumerate(events):
        arr[i] = None if e is None else e.cuda_event
    return arr


# ------------------------------------------------------------------------------- prefill
def _ptr_array(ts):
    arr = (C.c_void_p * len(ts))(*[None if t is None else t.data_ptr() for t in ts])
    return arr


def prefill_args(*, page_table, lens, max_len, host_keys, host_key_scales, summaries, block_scale,
                 host_kv=None, hbuf=None, pos_of_slot=None, slot_of_pos=None, recent_score=None) -> PrefillStreamArgs:
    """Per-layer lists: host_keys / host_key_scales / host_kv are pinned CPU tensors, the rest
    CUDA tensors; the hot-buffer lists are given together or not at all (no seeding)."""
    a = PrefillStreamArgs()
    a.layers = len(host_keys)
    a.batch = page_table.shape[0]
    a.max_pages = page_table.shape[1]
    a.max_len = int(max_len)
    a.max_blocks = summaries[0].shape[1]
    a.num_pages = host_keys[0].shape[0]
    seed = hbuf is not None
    a.n_slots = hbuf[0].shape[1] if seed else 0
    a.row_bytes = hbuf[0].shape[2] * hbuf[0].element_size() if seed else 0
    a.page_table, a.lens = _ptr(page_table), _ptr(lens)
    arrays = {"host_keys": host_keys, "host_key_scales": host_key_scales, "summaries": summaries,
              "block_scale": block_scale}
    if seed:
        arrays.update(host_kv=host_kv, hbuf=hbuf, pos_of_slot=pos_of_slot, slot_of_pos=slot_of_pos,
                      recent_score=recent_score)
    held = []
    for name, ts in arrays.items():
        arr = _ptr_array(ts)
        setattr(a, name, C.cast(arr, C.c_void_p).value)
        held.append(arr)
        held.extend(ts)
    return _hold(a, page_table, lens, *held)


def ls_prefill_stream_workspace_size(a: PrefillStreamArgs) -> int:
    return lib().ls_prefill_stream_workspace_size(C.byref(a))


def ls_prefill_stream(a: PrefillStreamArgs, workspace, stream=None):
    _check(lib().ls_prefill_stream(C.byref(a), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                   _stream(stream)))


# ------------------------------------------------------------------------------- context parallel
def cp_merge_args(*, cand_score, cand_pos, shard_begin, shard_end, idx, sel_score=None, local_sel=None):
    """cand_score / cand_pos: [G, B, k] gathered candidates (CUDA tensors)."""
    a = CpMergeArgs()
    a.shards, a.batch, a.k = cand_score.shape
    a.cand_score, a.cand_pos = _ptr(cand_score), _ptr(cand_pos)
    a.shard_begin, a.shard_end = _ptr(shard_begin), _ptr(shard_end)
    a.idx, a.sel_score, a.local_sel = _ptr(idx), _ptr(sel_score), _ptr(local_sel)
    return _hold(a, cand_score, cand_pos, shard_begin, shard_end, idx, sel_score, local_sel)


def ls_cp_merge_workspace_size(a: CpMergeArgs) -> int:
    return lib().ls_cp_merge_workspace_size(C.byref(a))


def ls_cp_merge_topk(a: CpMergeArgs, workspace, stream=None):
    _check(lib().ls_cp_merge_topk(C.byref(a), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                  _stream(stream)))


def ls_attn_merge(*, o_parts, lse_parts, o, lse, stream=None):
    """o_parts [G, B, H, dv] float32, lse_parts [G, B, H]; o [B, H, dv] bf16 or float32."""
    a = AttnMergeArgs()
    a.parts, a.batch, a.heads, a.dv = o_parts.shape
    a.o_parts, a.lse_parts, a.o, a.lse = _ptr(o_parts), _ptr(lse_parts), _ptr(o), _ptr(lse)
    a.o_dtype = LS_F32 if o.dtype == torch.float32 else LS_BF16
    _check(lib().ls_attn_merge(C.byref(a), _stream(stream)))


# ------------------------------------------------------------------------------- diagnostics
def ls_set_wait_limit(ns: int):
    _check(lib().ls_set_wait_limit(int(ns)))


def ls_selftest_bounded_wait(stream=None):
    _check(lib().ls_selftest_bounded_wait(_stream(stream)))
