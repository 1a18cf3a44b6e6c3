"""Stage-by-stage GPU parity against the CPU oracle, through the C ABI.

Every input comes from the seeded generators (never from a GPU stage); tolerances:
top-k and hot-buffer lists bit-exact (top-k: same fp32 scores on both sides),
attention max-abs 2e-2 for bf16 and 1e-4 for fp32, indexer scores 1e-3 * max|S|
(1e-4 for the fp32 path)."""
import math

import numpy as np
import pytest
import torch

import oracle.ls_oracle as O
from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import synthetic as syn

from gpu_helpers import (DEV, assert_status_clean, bits16, gpu_index_scores, oracle_index_inputs, round4)

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------- a1 indexer
def test_index_score_f32_tiny_config():
    inp = syn.indexer_f32([8192], heads=8, dim=64, seed=1001)
    got = gpu_index_scores(inp).cpu().numpy()
    ref = O.index_score(**oracle_index_inputs(inp))[0]
    assert np.abs(got[0, :8192] - ref).max() <= 1e-4 * np.abs(ref).max()


@pytest.mark.parametrize("variant", [0, 1])
def test_index_score_e4m3_ragged(variant):
    lens = [700, 64 * 64 + 17, 832, 64, 1]
    inp = syn.indexer_fp8(lens, seed=77)
    got = gpu_index_scores(inp, variant=variant).cpu().numpy()
    ref = O.index_score(**oracle_index_inputs(inp))
    for b, L in enumerate(lens):
        r = ref[b]
        assert np.abs(got[b, :L] - r).max() <= 1e-3 * max(np.abs(r).max(), 1e-30), b
        assert np.isnan(got[b, L:]).all(), "positions >= L must stay untouched"
    assert_status_clean()


def test_index_score_tc_matches_cuda_core_kernel():
    inp = syn.indexer_fp8([5000, 12345], seed=78)
    a = gpu_index_scores(inp, variant=0).cpu().numpy()
    b = gpu_index_scores(inp, variant=1).cpu().numpy()
    for i, L in enumerate(inp.lens.tolist()):
        assert np.abs(a[i, :L] - b[i, :L]).max() <= 1e-4 * np.abs(b[i, :L]).max()


def test_index_score_bad_page_is_flagged_not_read():
    inp = syn.indexer_fp8([256], seed=79)
    inp.page_table[0, 2] = 10 ** 6  # beyond the pool
    got = gpu_index_scores(inp).cpu().numpy()
    assert np.isnan(got[0, 128:192]).all()
    assert B.ls_check_device_status() & B.LS_DEV_BOUNDS


# ----------------------------------------------------------------------------- a2 top-k
def _topk_case(lens, k, seed, kind="normal"):
    g = torch.Generator().manual_seed(seed)
    ml = round4(max(lens))
    if kind == "ties":
        s = torch.randint(-4, 5, (len(lens), ml), generator=g).float() * 0.5
    elif kind == "zeros":
        s = torch.randint(0, 3, (len(lens), ml), generator=g).float() - 1.0
        s = torch.where(s == 0, torch.where(torch.rand(s.shape, generator=g) < 0.5, -0.0, 0.0), s)
    elif kind in ("ascending", "descending"):
        # the largest scores bunched at one end of the request
        s = torch.arange(ml, dtype=torch.float32)[None].repeat(len(lens), 1)
        s = s if kind == "ascending" else -s
    else:
        s = torch.randn((len(lens), ml), generator=g)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    idx = torch.full((len(lens), k), -7, dtype=torch.int32, device=DEV)
    sel = torch.zeros((len(lens), k), device=DEV)
    B.ls_topk_select(scores=s.to(DEV), lens=lens_t.to(DEV), idx=idx, sel_score=sel)
    torch.cuda.synchronize()
    idx, sel = idx.cpu().numpy(), sel.cpu().numpy()
    sn = s.numpy()
    for b, L in enumerate(lens):
        ref, _ = O.topk_select(sn[b, :L].astype(np.float64), k)
        assert np.array_equal(idx[b], ref), (b, L)
        n = min(k, L)
        assert np.array_equal(sel[b, :n], sn[b, ref[:n]]) or kind == "zeros"
    assert_status_clean()


@pytest.mark.parametrize("lens,k", [([10, 2048, 5000, 131072, 300], 2048), ([8192], 256), ([1000, 999], 1),
                                    ([70000, 4096], 4096)])
def test_topk_exact(lens, k):
    _topk_case(lens, k, seed=sum(lens) + k)


@pytest.mark.parametrize("kind", ["ties", "zeros"])
def test_topk_ties_lower_position_first(kind):
    _topk_case([3000, 40000, 129], 512, seed=5, kind=kind)


@pytest.mark.parametrize("kind", ["ascending", "descending"])
@pytest.mark.parametrize("lens", [[32768, 20001, 6000], [131072, 70001, 6000]])
def test_topk_bunched_scores(kind, lens):
    # the top keys of a request share a few segments: (short requests) the per-segment
    # lists of the one-CTA kernel overflow and it finishes from the scores; (long ones) the
    # cluster kernel's candidate buffers overflow into its general path
    _topk_case(lens, 2048, seed=7, kind=kind)


@pytest.mark.parametrize("kind", ["ties", "zeros"])
def test_topk_ties_short_requests(kind):
    # the one-CTA kernel (every request at most 32,768 scores)
    _topk_case([3000, 20000, 129, 32768], 512, seed=6, kind=kind)


def test_topk_full_scan_1m_context():
    # slices larger than the shared-memory cache take the global-memory path
    _topk_case([1 << 20, (1 << 20) - 5], 2048, seed=9)


def test_topk_permutation_identity_on_gpu():
    g = torch.Generator().manual_seed(3)
    s = torch.randn((1, 65536), generator=g)
    perm = torch.randperm(65536, generator=g)
    lens = torch.tensor([65536], dtype=torch.int32, device=DEV)
    out = []
    for x in (s, s[:, perm]):
        idx = torch.empty((1, 2048), dtype=torch.int32, device=DEV)
        B.ls_topk_select(scores=x.contiguous().to(DEV), lens=lens, idx=idx)
        out.append(idx.cpu().numpy()[0])
    assert sorted(perm.numpy()[out[1]].tolist()) == out[0].tolist()


# ----------------------------------------------------------------------------- a6 attention
def _random_selection(B_, k, L, seed, n_valid=None):
    g = torch.Generator().manual_seed(seed)
    sel = torch.full((B_, k), -1, dtype=torch.int32)
    for b in range(B_):
        n = k if n_valid is None else n_valid[b]
        pos = torch.randperm(L[b] if isinstance(L, list) else L, generator=g)[:n].sort().values
        sel[b, :n] = pos.to(torch.int32)
    return sel


def _oracle_attn(q_bits, pool_bits, pt, sel, scale, dv):
    out_o, out_l = [], []
    for b in range(q_bits.shape[0]):
        rows = O.bf16_decode(O.selected_rows(pool_bits, pt[b], sel[b]))
        o, l = O.sparse_attn_decode(O.bf16_decode(q_bits[b]), rows, rows[:, :dv], scale)
        out_o.append(o)
        out_l.append(l)
    return np.stack(out_o), np.stack(out_l)


@pytest.mark.parametrize("variant,scale", [(0, 1 / math.sqrt(576)), (1, 1 / math.sqrt(576)), (0, 0.25)])
def test_mla_attention_paged(variant, scale):
    lens = [20000, 9000, 4096]
    Bn, k = 3, 2048
    table, n_pool = syn.page_layout(lens, seed=11)
    q, kv = syn.mla_attention(Bn, n_pool, seed=12)
    sel = _random_selection(Bn, k, lens, seed=13, n_valid=[2048, 1500, 17])
    o = torch.zeros((Bn, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros((Bn, 128), device=DEV)
    a = B.attn_args(q=q.to(DEV), k_rows=kv.to(DEV), sel=sel.to(DEV), o=o, lse=lse, scale=scale,
                    page_table=table.to(DEV), variant=variant)
    ws = torch.empty(max(1, B.ls_sparse_attn_workspace_size(a)), dtype=torch.uint8, device=DEV)
    B.ls_sparse_attn_decode(a, ws)
    torch.cuda.synchronize()
    ref_o, ref_l = _oracle_attn(bits16(q), bits16(kv), table.numpy(), sel.numpy(), scale, 512)
    assert np.abs(o.float().cpu().numpy() - ref_o).max() <= 2e-2
    assert np.abs(lse.cpu().numpy() - ref_l).max() <= 2e-2
    assert_status_clean()


@pytest.mark.parametrize("lens,k,n_valid", [
    ([3000, 700], 100, [100, 37]),        # two tiles: one KV split, the output written by the attention itself
    ([70000, 5000], 4096, [4096, 3000]),  # the largest k: 64 tiles
])
def test_mla_attention_split_extremes(lens, k, n_valid):
    Bn = len(lens)
    table, n_pool = syn.page_layout(lens, seed=21)
    q, kv = syn.mla_attention(Bn, n_pool, seed=22)
    sel = _random_selection(Bn, k, lens, seed=23, n_valid=n_valid)
    scale = 1 / math.sqrt(576)
    o = torch.zeros((Bn, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros((Bn, 128), device=DEV)
    a = B.attn_args(q=q.to(DEV), k_rows=kv.to(DEV), sel=sel.to(DEV), o=o, lse=lse, scale=scale,
                    page_table=table.to(DEV))
    ws = torch.empty(max(1, B.ls_sparse_attn_workspace_size(a)), dtype=torch.uint8, device=DEV)
    B.ls_sparse_attn_decode(a, ws)
    torch.cuda.synchronize()
    ref_o, ref_l = _oracle_attn(bits16(q), bits16(kv), table.numpy(), sel.numpy(), scale, 512)
    assert np.abs(o.float().cpu().numpy() - ref_o).max() <= 2e-2
    assert np.abs(lse.cpu().numpy() - ref_l).max() <= 2e-2
    assert_status_clean()


@pytest.mark.parametrize("Bn,heads_step", [
    (8, 4),    # 8 KV splits: the splits of a request merge in one 16-CTA cluster
    (15, 8),   # 4 splits: an 8-CTA cluster
    (30, 16),  # 2 splits: a 4-CTA cluster
    (10, 8),   # 7 splits: partials through the workspace and the combine kernel
])
def test_mla_attention_batch_sizes_and_split_merges(Bn, heads_step):
    """Batch sizes whose KV split counts take each way of merging the splits: inside the
    cluster (2, 4, 8 splits) or through the workspace (7); ragged and empty selections
    included.  Heads sampled every `heads_step` for the oracle."""
    L, k = 8192, 2048
    lens = [L] * Bn
    table, n_pool = syn.page_layout(lens, seed=31 + Bn)
    q, kv = syn.mla_attention(Bn, n_pool, seed=32 + Bn)
    n_valid = [k] * Bn
    n_valid[1] = 1111
    n_valid[Bn - 1] = 0  # an empty selection: o = 0, lse = -inf
    sel = _random_selection(Bn, k, lens, seed=33 + Bn, n_valid=n_valid)
    scale = 1 / math.sqrt(576)
    o = torch.full((Bn, 128, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((Bn, 128), float("nan"), device=DEV)
    a = B.attn_args(q=q.to(DEV), k_rows=kv.to(DEV), sel=sel.to(DEV), o=o, lse=lse, scale=scale,
                    page_table=table.to(DEV))
    ws = torch.empty(max(1, B.ls_sparse_attn_workspace_size(a)), dtype=torch.uint8, device=DEV)
    B.ls_sparse_attn_decode(a, ws)
    torch.cuda.synchronize()
    hs = slice(0, 128, heads_step)
    qb, kvb = bits16(q), bits16(kv)
    for b in range(Bn - 1):
        rows = O.bf16_decode(O.selected_rows(kvb, table.numpy()[b], sel.numpy()[b]))
        ref_o, ref_l = O.sparse_attn_decode(O.bf16_decode(qb[b][hs]), rows, rows[:, :512], scale)
        assert np.abs(o[b][hs].float().cpu().numpy() - ref_o).max() <= 2e-2, b
        assert np.abs(lse[b][hs].cpu().numpy() - ref_l).max() <= 2e-2, b
    assert (o[Bn - 1].float() == 0).all() and torch.isneginf(lse[Bn - 1]).all()
    assert_status_clean()


def test_mla_attention_slots_and_empty_selection():
    Bn, S, k = 2, 4096, 64
    g = torch.Generator().manual_seed(21)
    hbuf = torch.randn((Bn, S, 576), generator=g).to(torch.bfloat16)
    q = torch.randn((Bn, 128, 576), generator=g).to(torch.bfloat16)
    sel = torch.full((Bn, k), -1, dtype=torch.int32)
    sel[0] = torch.randperm(S, generator=g)[:k].to(torch.int32)  # slots need not be sorted
    o = torch.zeros((Bn, 128, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros((Bn, 128), device=DEV)
    a = B.attn_args(q=q.to(DEV), k_rows=hbuf.to(DEV), sel=sel.to(DEV), o=o, lse=lse, scale=1 / 24,
                    n_slots=S)
    ws = torch.empty(max(1, B.ls_sparse_attn_workspace_size(a)), dtype=torch.uint8, device=DEV)
    B.ls_sparse_attn_decode(a, ws)
    torch.cuda.synchronize()
    rows = O.bf16_decode(bits16(hbuf[0][sel[0].long()]))
    ref_o, ref_l = O.sparse_attn_decode(O.bf16_decode(bits16(q[0])), rows, rows[:, :512], 1 / 24)
    assert np.abs(o[0].float().cpu().numpy() - ref_o).max() <= 2e-2
    assert np.abs(lse[0].cpu().numpy() - ref_l).max() <= 2e-2
    # request 1 selected nothing: o = 0, lse = -inf
    assert (o[1].float() == 0).all() and torch.isneginf(lse[1]).all()
    assert_status_clean()


def test_f32_attention_tiny_config():
    L, k = 8192, 256
    table = torch.arange(128, dtype=torch.int32)[None]
    q, K, V = syn.f32_attention(1, 128, heads=16, d=128, seed=2001)
    sel = _random_selection(1, k, L, seed=22)
    o = torch.zeros((1, 16, 128), device=DEV)
    lse = torch.zeros((1, 16), device=DEV)
    a = B.attn_args(q=q.to(DEV), k_rows=K.to(DEV), v_rows=V.to(DEV), sel=sel.to(DEV), o=o, lse=lse,
                    scale=1 / math.sqrt(128), page_table=table.to(DEV))
    B.ls_sparse_attn_decode(a, None)
    torch.cuda.synchronize()
    kr = O.selected_rows(K.numpy().astype(np.float64), table[0].numpy(), sel[0].numpy())
    vr = O.selected_rows(V.numpy().astype(np.float64), table[0].numpy(), sel[0].numpy())
    ref_o, ref_l = O.sparse_attn_decode(q[0].double().numpy(), kr, vr, 1 / math.sqrt(128))
    assert np.abs(o[0].cpu().numpy() - ref_o).max() <= 1e-4
    assert np.abs(lse[0].cpu().numpy() - ref_l).max() <= 1e-4


# ----------------------------------------------------------------------------- a4/a5 hot buffer
def _hotbuf_case(lens, k, miss_frac, seed, n_slots=4096, partial_fill=False):
    Bn = len(lens)
    ml = round4(max(lens))
    sel = _random_selection(Bn, k, lens, seed=seed)
    pos_of_slot, slot_of_pos, recent = syn.hot_buffer_state([s[s >= 0] for s in sel], lens, n_slots=n_slots,
                                                            miss_frac=miss_frac, seed=seed + 1, max_len=ml)
    if partial_fill:  # empty some slots and plant score ties
        for b in range(Bn):
            drop = torch.nonzero(pos_of_slot[b] >= 0).flatten()[::3]
            keep_sel = set(sel[b].tolist())
            for s in drop.tolist():
                p = int(pos_of_slot[b, s])
                if p not in keep_sel:
                    slot_of_pos[b, p] = -1
                    pos_of_slot[b, s] = -1
        recent = (recent * 4).floor() / 4
    g = torch.Generator().manual_seed(seed + 2)
    sel_score = torch.randn((Bn, k), generator=g)
    return sel, sel_score, pos_of_slot, slot_of_pos, recent


@pytest.mark.parametrize("miss_frac,partial", [(0.2, False), (0.4, False), (0.3, True)])
def test_hotbuf_resolve_and_gather_exact(miss_frac, partial):
    lens = [131072, 60000, 9000]
    Bn, k, S = 3, 2048, 4096
    sel, sel_score, pos_of_slot, slot_of_pos, recent = _hotbuf_case(lens, k, miss_frac, 31, S, partial)
    d = dict(sel=sel.to(DEV), sel_score=sel_score.to(DEV), pos_of_slot=pos_of_slot.to(DEV),
             recent_score=recent.to(DEV), slot_of_pos=slot_of_pos.to(DEV))
    outs = dict(sel_slot=torch.empty((Bn, k), dtype=torch.int32, device=DEV),
                miss_pos=torch.empty((Bn, k), dtype=torch.int32, device=DEV),
                miss_slot=torch.empty((Bn, k), dtype=torch.int32, device=DEV),
                n_miss=torch.empty((Bn,), dtype=torch.int32, device=DEV))
    B.ls_hotbuf_resolve(**d, **outs)
    # gather: history in pinned host memory, hot buffer in HBM
    table, n_pool = syn.page_layout(lens, seed=32)
    g = torch.Generator().manual_seed(33)
    host = torch.randint(-32768, 32767, (n_pool, 64, 576), generator=g, dtype=torch.int16).pin_memory()
    hbuf0 = torch.randint(-32768, 32767, (Bn, S, 576), generator=g, dtype=torch.int16)
    hbuf = hbuf0.to(DEV)
    B.ls_gather_misses(host_kv=host, page_table=table.to(DEV), miss_pos=outs["miss_pos"],
                       miss_slot=outs["miss_slot"], n_miss=outs["n_miss"], hbuf=hbuf)
    torch.cuda.synchronize()
    for b in range(Bn):
        r = O.hotbuf_resolve(sel[b].numpy(), sel_score[b].numpy(), pos_of_slot[b].numpy(), recent[b].numpy(),
                             slot_of_pos[b].numpy())
        assert np.array_equal(outs["sel_slot"][b].cpu().numpy(), r["sel_slot"])
        assert np.array_equal(outs["miss_pos"][b].cpu().numpy(), r["miss_pos"])
        assert np.array_equal(outs["miss_slot"][b].cpu().numpy(), r["miss_slot"])
        assert int(outs["n_miss"][b]) == r["n_miss"]
        assert np.array_equal(d["pos_of_slot"][b].cpu().numpy(), r["pos_of_slot"])
        assert np.array_equal(d["slot_of_pos"][b].cpu().numpy(), r["slot_of_pos"])
        assert np.array_equal(d["recent_score"][b].cpu().numpy(), r["recent_score"])
        ref_h = O.gather_misses(host.numpy(), table[b].numpy(), r["miss_pos"], r["miss_slot"], r["n_miss"],
                                hbuf0[b].numpy())
        assert np.array_equal(hbuf[b].cpu().numpy(), ref_h)
    assert_status_clean()


# ----------------------------------------------------------------------------- a3 coarse-to-fine
def _c2f_inputs(lens, seed, clustered=True, sigma=0.05, w_mixed=False):
    """Coarse-to-fine indexer inputs: block-clustered keys (2% of the blocks shifted toward
    the query) or i.i.d. keys; head weights >= 0, or of both signs with ``w_mixed``."""
    Bn = len(lens)
    g = torch.Generator().manual_seed(seed)
    qf = torch.randn((Bn, 64, 128), generator=g)
    table, n_pool = syn.page_layout(lens, seed + 17)
    if clustered:
        w = (torch.randn((Bn, 64), generator=g) * 0.1).abs()
        direction = (w[:, :, None] * qf).sum(1)
        keys = torch.cat([syn.clustered_keys(-(-L // 64), 1, within_sigma=sigma, direction=direction[b:b + 1],
                                             seed=seed + b)[:L] for b, L in enumerate(lens)])
    else:
        keys = torch.randn((sum(lens), 128), generator=g)
    pool_keys = syn.logical_to_pool(keys, lens, table, n_pool)
    inp = syn.indexer_fp8(lens, seed=seed, w_nonneg=not w_mixed, q=qf, keys=pool_keys)
    return inp


def test_block_summaries_exact():
    lens = [64 * 300 + 17, 64 * 41]
    inp = _c2f_inputs(lens, seed=41)
    d = {k: v.to(DEV) for k, v in inp.__dict__.items() if isinstance(v, torch.Tensor)}
    mb = max(-(-L // 64) for L in lens)
    summ = torch.zeros((2, mb, 256), dtype=torch.uint8, device=DEV)
    bsc = torch.zeros((2, mb), device=DEV)
    B.ls_build_block_summaries(q=d["q"], w=d["w"], key_pool=d["key_pool"], key_scale=d["key_scale"],
                               q_scale=d["q_scale"], page_table=d["page_table"], lens=d["lens"],
                               max_len=round4(max(lens)), summaries=summ, block_scale=bsc)
    torch.cuda.synchronize()
    for b, L in enumerate(lens):
        kmax8, kmin8, bs = O.block_summaries(inp.key_pool.numpy(), inp.key_scale.numpy(),
                                             inp.page_table.numpy()[b], L)
        nb = kmax8.shape[0]
        assert np.array_equal(summ[b, :nb, :128].cpu().numpy(), kmax8)
        assert np.array_equal(summ[b, :nb, 128:].cpu().numpy(), kmin8)
        assert np.array_equal(bsc[b, :nb].cpu().numpy(), bs)
    assert_status_clean()


def run_c2f(inp, k, eps_rel=0.0, keys_on_host=False, stage_blocks=0):
    lens = inp.lens.tolist()
    Bn = len(lens)
    d = {kk: v.to(DEV) for kk, v in inp.__dict__.items() if isinstance(v, torch.Tensor)}
    mb = max(-(-L // 64) for L in lens)
    ml = round4(max(lens))
    summ = torch.zeros((Bn, mb, 256), dtype=torch.uint8, device=DEV)
    bsc = torch.zeros((Bn, mb), device=DEV)
    B.ls_build_block_summaries(q=d["q"], w=d["w"], key_pool=d["key_pool"], key_scale=d["key_scale"],
                               q_scale=d["q_scale"], page_table=d["page_table"], lens=d["lens"], max_len=ml,
                               summaries=summ, block_scale=bsc)
    keys, kscale = d["key_pool"], d["key_scale"]
    if keys_on_host:  # the summaries came from the device copy; scoring reads the host copy
        keys, kscale = inp.key_pool.pin_memory(), inp.key_scale.pin_memory()
        del d["key_pool"], d["key_scale"]
    ix = B.index_args(q=d["q"], w=d["w"], key_pool=keys, page_table=d["page_table"], lens=d["lens"],
                      q_scale=d["q_scale"], key_scale=kscale, max_len=ml)
    idx = torch.full((Bn, k), -7, dtype=torch.int32, device=DEV)
    sel = torch.zeros((Bn, k), device=DEV)
    surv = torch.full((Bn, mb), -1, dtype=torch.int32, device=DEV)
    nsurv = torch.zeros((Bn,), dtype=torch.int32, device=DEV)
    ub = torch.full((Bn, mb), float("nan"), device=DEV)
    a = B.c2f_args(index=ix, k=k, summaries=summ, block_scale=bsc, idx=idx, sel_score=sel, survivors=surv,
                   n_survivors=nsurv, ub=ub, eps_rel=eps_rel, keys_on_host=keys_on_host, stage_blocks=stage_blocks)
    ws = torch.empty(B.ls_block_bound_prune_workspace_size(a), dtype=torch.uint8, device=DEV)
    B.ls_block_bound_prune(a, ws)
    torch.cuda.synchronize()
    return idx, sel, surv, nsurv, ub


@pytest.mark.parametrize("clustered,lens,k", [(True, [64 * 4000 + 5, 64 * 2500], 2048),
                                               (False, [64 * 700 + 33], 2048),
                                               (True, [1500, 64 * 900], 2048)])
def test_c2f_equals_full_scan(clustered, lens, k):
    inp = _c2f_inputs(lens, seed=51, clustered=clustered)
    idx, sel, surv, nsurv, ub = run_c2f(inp, k)
    # GPU full scan on the same inputs
    scores = gpu_index_scores(inp)
    full = torch.empty((len(lens), k), dtype=torch.int32, device=DEV)
    B.ls_topk_select(scores=scores, lens=inp.lens.to(DEV), idx=full)
    torch.cuda.synchronize()
    assert torch.equal(idx, full), "coarse-to-fine must return exactly the full-scan top-k"
    ref = O.index_score(**oracle_index_inputs(inp))
    for b, L in enumerate(lens):
        check_topk_band_local(idx[b].cpu().numpy(), ref[b], k)
        n = int(nsurv[b])
        blocks = set(surv[b, :n].cpu().numpy().tolist())
        chosen = idx[b].cpu().numpy()
        assert set((chosen[chosen >= 0] // 64).tolist()) <= blocks
        if clustered and L > 64 * 1000:
            assert n < 0.5 * (-(-L // 64)), f"clustered keys should prune (kept {n})"
        # the plain bound dominates every GPU score of its block
        s = scores[b, :L].cpu().numpy()
        u = ub[b, :-(-L // 64)].cpu().numpy()
        blockmax = np.array([s[j * 64:(j + 1) * 64].max() for j in range(u.shape[0])])
        assert (u >= blockmax - 1e-4 * np.abs(blockmax).max()).all()
    assert_status_clean()


@pytest.mark.parametrize("clustered,lens,stage", [(True, [64 * 4000 + 5, 64 * 2500], 0),
                                                   (False, [64 * 700 + 33], 64),
                                                   (True, [1500, 64 * 900 + 9], 40)])
def test_c2f_host_keys_same_as_device_keys(clustered, lens, stage):
    """Keys in pinned host memory, fetched block by block into staging (several passes
    when the survivors outnumber the staging): the same selection, scores, survivors and
    bounds as with the keys in HBM."""
    inp = _c2f_inputs(lens, seed=61, clustered=clustered)
    ref = run_c2f(inp, 2048)
    got = run_c2f(inp, 2048, keys_on_host=True, stage_blocks=stage)
    names = ("idx", "sel_score", "survivors", "n_survivors", "ub")
    for name, r, g in zip(names, ref, got):
        assert torch.equal(r.nan_to_num(-9.0), g.nan_to_num(-9.0)), name
    if not clustered:  # every block survives: the survivors took many staging passes
        assert int(got[3][0]) > 4 * 64
    assert_status_clean()


def test_c2f_host_keys_rejects_device_keys():
    inp = _c2f_inputs([64 * 200], seed=62)
    d = {kk: v.to(DEV) for kk, v in inp.__dict__.items() if isinstance(v, torch.Tensor)}
    ix = B.index_args(q=d["q"], w=d["w"], key_pool=d["key_pool"], page_table=d["page_table"], lens=d["lens"],
                      q_scale=d["q_scale"], key_scale=d["key_scale"], max_len=64 * 200)
    summ = torch.zeros((1, 200, 256), dtype=torch.uint8, device=DEV)
    bsc = torch.ones((1, 200), device=DEV)
    idx = torch.zeros((1, 2048), dtype=torch.int32, device=DEV)
    a = B.c2f_args(index=ix, k=2048, summaries=summ, block_scale=bsc, idx=idx, keys_on_host=True)
    ws = torch.empty(B.ls_block_bound_prune_workspace_size(a), dtype=torch.uint8, device=DEV)
    with pytest.raises(B.LsError, match="pinned host memory"):
        B.ls_block_bound_prune(a, ws)


@pytest.mark.parametrize("clustered,w_mixed", [(True, False), (False, False), (True, True)])
def test_block_bound_matches_oracle(clustered, w_mixed):
    """The bound the GPU prunes with (without its margin) against the oracle's block bound
    from the same stored summaries: equal to within fp32 rounding, which is held to 2^-12 of
    the block's magnitude bound M_j = 448 bs_j sum_h |w_h sq_h| sum_d |q_hd| -- a quarter of
    the 2^-10 M_j margin the pruning adds, so the margin covers the rounding; a dropped head
    or dim, a sign or a scale slip moves the bound by far more.  With head weights of both
    signs the bound uses the lower box end for w_h < 0."""
    lens = [64 * 900 + 21, 64 * 300]
    inp = _c2f_inputs(lens, seed=71, clustered=clustered, w_mixed=w_mixed)
    if w_mixed:
        assert (inp.w.float() < 0).any() and (inp.w.float() > 0).any()
    idx, sel, surv, nsurv, ub = run_c2f(inp, 2048)
    wb = inp.w.view(torch.int16).numpy().view(np.uint16)
    for b, L in enumerate(lens):
        kmax8, kmin8, bs = O.block_summaries(inp.key_pool.numpy(), inp.key_scale.numpy(),
                                             inp.page_table.numpy()[b], L)
        ref = O.block_bound(inp.q[b].numpy(), inp.q_scale[b].numpy(), wb[b], kmax8, kmin8, bs)
        qabs = np.abs(O.e4m3_decode(inp.q[b].numpy())).sum(axis=1)          # [H]
        wsq = np.abs(O.bf16_decode(wb[b]) * inp.q_scale[b].numpy().astype(np.float64))
        mag = 448.0 * bs.astype(np.float64) * float((wsq * qabs).sum())     # [NB]
        got = ub[b, :ref.shape[0]].cpu().numpy().astype(np.float64)
        err = np.abs(got - ref)
        assert (err <= 2.0 ** -12 * mag).all(), float((err / mag).max())
        assert (ref > 0).any()
    assert_status_clean()


def test_c2f_million_token_context_against_oracle():
    """The coarse-to-fine indexer at the 1,048,576-token context of its workload (one
    request): the selection lies within the tie band of the oracle's full-scan top-k,
    equals the GPU's own full scan, comes only from surviving blocks, and pruning
    happened."""
    lens = [1048576]
    k = 2048
    inp = _c2f_inputs(lens, seed=81, clustered=True)
    idx, sel, surv, nsurv, ub = run_c2f(inp, k)
    ref = O.index_score(**oracle_index_inputs(inp))[0]
    g = idx[0].cpu().numpy()
    check_topk_band_local(g, ref, k)
    s = sel[0].cpu().numpy()
    assert np.abs(s - ref[g]).max() <= 1e-3 * np.abs(ref).max()
    scores = gpu_index_scores(inp)
    full = torch.empty((1, k), dtype=torch.int32, device=DEV)
    B.ls_topk_select(scores=scores, lens=inp.lens.to(DEV), idx=full)
    torch.cuda.synchronize()
    assert torch.equal(idx, full)
    n = int(nsurv[0])
    assert n < 0.25 * (lens[0] // 64), f"clustered keys should prune (kept {n} of {lens[0] // 64})"
    assert set((g // 64).tolist()) <= set(surv[0, :n].cpu().numpy().tolist())
    assert_status_clean()


def check_topk_band_local(g, s, k):
    from gpu_helpers import check_topk_band
    check_topk_band(g, s, k)
