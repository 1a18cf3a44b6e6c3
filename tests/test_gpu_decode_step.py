"""End-to-end ls_decode_step parity against the CPU oracle on every workload shape:
the fp32 tiny config, the MLA batch at 128K (reduced, and at full size in the launch
configuration the benchmark times), hot-buffer decode with 20% / 40% misses, the
coarse-to-fine indexer at long context, and a ragged mixed batch."""
import math

import numpy as np
import pytest
import torch

import oracle.ls_oracle as O
from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import synthetic as syn
from sparse_attention_decode_ls_b200 import workload as W

from gpu_helpers import DEV, assert_status_clean, bits16, check_topk_band, gpu_index_scores, oracle_index_inputs

pytestmark = pytest.mark.gpu


def _oracle_selection(inp, k):
    scores = O.index_score(**oracle_index_inputs(inp))
    idx = np.stack([O.topk_select(s, k)[0] for s in scores])
    sel = np.stack([O.topk_select(s, k)[1] for s in scores])
    return scores, idx, sel


def _check_mla_step(wl, inp, q, kv, k, heads_sample=None):
    """Run the step; every request's selection must lie within the tie band of the oracle's,
    and the step's own output is compared with the oracle's attention over that (validated)
    selection, so the comparison never depends on the two selections coinciding."""
    wl.step()
    torch.cuda.synchronize()
    assert_status_clean()
    scores, ref_idx, _ = _oracle_selection(inp, k)
    gidx = wl.idx.cpu().numpy()
    for b in range(wl.batch):
        check_topk_band(gidx[b], scores[b], k)
    qb, kvb = bits16(q), bits16(kv)
    pt = inp.page_table.numpy()
    o_gpu = wl.o.float().cpu().numpy()
    l_gpu = wl.lse.cpu().numpy()
    hs = slice(None) if heads_sample is None else heads_sample
    for b in range(wl.batch):
        rows = O.bf16_decode(O.selected_rows(kvb, pt[b], gidx[b]))
        o, l = O.sparse_attn_decode(O.bf16_decode(qb[b][hs]), rows, rows[:, :512], syn.softmax_scale(576))
        assert np.abs(o_gpu[b][hs] - o).max() <= 2e-2, b
        assert np.abs(l_gpu[b][hs] - l).max() <= 2e-2, b


def test_decode_step_tiny_f32():
    """The fp32 configuration: the selection within the tie band of the oracle's, and the
    attention always checked at 1e-4 against the oracle on the GPU's own selection (which the
    band check has just validated), whether or not the two selections coincide."""
    wl = W.tiny_f32()
    wl.step()
    torch.cuda.synchronize()
    assert_status_clean()
    inp = syn.indexer_f32([8192], heads=8, dim=64, seed=1001)
    q, K, V = syn.f32_attention(1, 128, heads=16, d=128, seed=2001)
    scores, ref_idx, _ = _oracle_selection(inp, 256)
    gidx = wl.idx.cpu().numpy()[0]
    check_topk_band(gidx, scores[0], 256)
    pt = inp.page_table.numpy()[0]
    kr = O.selected_rows(K.numpy().astype(np.float64), pt, gidx)
    vr = O.selected_rows(V.numpy().astype(np.float64), pt, gidx)
    o, l = O.sparse_attn_decode(q[0].double().numpy(), kr, vr, 1 / math.sqrt(128))
    assert np.abs(wl.o.cpu().numpy()[0] - o).max() <= 1e-4
    assert np.abs(wl.lse.cpu().numpy()[0] - l).max() <= 1e-4
    # the selection scores the step returns are the indexer's scores of the chosen positions
    gsel = wl.tensors["sel"].cpu().numpy()[0]
    assert np.abs(gsel - scores[0][gidx]).max() <= 1e-4 * np.abs(scores[0]).max()


def test_decode_step_mla_reduced():
    lens = [20000, 20000]
    inp = syn.indexer_fp8(lens, seed=301)
    q, kv = syn.mla_attention(2, inp.key_pool.shape[0], seed=302)
    wl = W.build("mla_reduced", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)))
    _check_mla_step(wl, inp, q, kv, 2048)


def test_decode_step_mla_full_size_bench_config():
    """B=8 at 131,072 tokens, k=2,048: the configuration bench.py times.  Scores and
    selections are checked for every request; attention on a sample of 16 heads."""
    lens = [131072] * 8
    inp = syn.indexer_fp8(lens, seed=1002)
    q, kv = syn.mla_attention(8, inp.key_pool.shape[0], seed=2002)
    wl = W.build("mla_full", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)))
    _check_mla_step(wl, inp, q, kv, 2048, heads_sample=slice(0, 128, 8))


def _hotbuf_step(lens, miss_frac, seed):
    """One hot-buffer decode step (history in pinned host memory, overlapped miss path),
    every request checked against the oracle: the selection within the tie band; the
    resolve's lists, counts, maps and recent scores bit for bit, and the whole post-step hot
    buffer byte for byte, against the oracle's resolve and gather run on the GPU's own
    (band-validated) selection and scores; attention against the oracle on that selection."""
    Bn, k = len(lens), 2048
    inp = syn.indexer_fp8(lens, seed=seed)
    scores, ref_idx, ref_sel = _oracle_selection(inp, k)
    ml = (max(lens) + 3) // 4 * 4
    pos_of_slot, slot_of_pos, recent = syn.hot_buffer_state([r[r >= 0] for r in ref_idx], lens, n_slots=4096,
                                                            miss_frac=miss_frac, seed=seed + 1, max_len=ml)
    n_pool = inp.key_pool.shape[0]
    q, kv = syn.mla_attention(Bn, n_pool, seed=seed + 2)
    host = kv.view(torch.int16).pin_memory()
    wl = W.build("hotbuf", inp, k=k, attn=dict(q=q, kv_host=True, scale=syn.softmax_scale(576)),
                 hotbuf=dict(pos_of_slot=pos_of_slot, slot_of_pos=slot_of_pos, recent=recent,
                             host_kv=host.view(torch.bfloat16)))
    hbuf0 = wl.hotbuf_init["hbuf"].view(torch.int16).cpu().numpy().view(np.uint16)
    wl.step()
    torch.cuda.synchronize()
    assert_status_clean()
    t = wl.tensors
    gidx = wl.idx.cpu().numpy()
    gsel = t["sel"].cpu().numpy()
    qb = bits16(q)
    kvb = bits16(kv)
    pt = inp.page_table.numpy()
    hb = t["hbuf"].view(torch.int16).cpu().numpy().view(np.uint16)
    same_as_oracle = 0
    for b in range(Bn):
        check_topk_band(gidx[b], scores[b], k)
        valid = gidx[b] >= 0
        assert np.abs(gsel[b][valid] - scores[b][gidx[b][valid]]).max() <= 1e-3 * np.abs(scores[b]).max()
        r = O.hotbuf_resolve(gidx[b], gsel[b], pos_of_slot[b].numpy(), recent[b].numpy(), slot_of_pos[b].numpy())
        for key in ("sel_slot", "miss_pos", "miss_slot"):
            assert np.array_equal(t[key][b].cpu().numpy(), r[key]), (b, key)
        assert int(t["n_miss"][b]) == r["n_miss"], b
        for key in ("pos_of_slot", "slot_of_pos", "recent_score"):
            assert np.array_equal(t[key][b].cpu().numpy(), r[key]), (b, key)
        if np.array_equal(gidx[b], ref_idx[b]):
            same_as_oracle += 1
            assert r["n_miss"] == int(round(miss_frac * k))  # the workload's planted miss rate
        # the whole hot buffer after the step: resident rows untouched, every miss's row
        # copied from the history into its victim slot
        ref_h = O.gather_misses(kvb, pt[b], r["miss_pos"], r["miss_slot"], r["n_miss"], hbuf0[b])
        assert np.array_equal(hb[b], ref_h), b
        rows = O.bf16_decode(O.selected_rows(kvb, pt[b], gidx[b]))
        o, l = O.sparse_attn_decode(O.bf16_decode(qb[b]), rows, rows[:, :512], syn.softmax_scale(576))
        assert np.abs(wl.o[b].float().cpu().numpy() - o).max() <= 2e-2
        assert np.abs(wl.lse[b].cpu().numpy() - l).max() <= 2e-2
    assert same_as_oracle >= 1  # the planted miss rate was seen on at least one request


@pytest.mark.parametrize("miss_frac", [0.2, 0.4])
def test_decode_step_hot_buffer(miss_frac):
    _hotbuf_step([131072, 131072], miss_frac, seed=401)


def test_decode_step_ragged_hot_buffer():
    lens = syn.ragged_lens(6, seed=1005)
    _hotbuf_step(lens, 0.2, seed=501)


def test_decode_step_coarse_to_fine():
    from test_gpu_stages import _c2f_inputs
    lens = [64 * 8192, 64 * 5000 + 7]
    inp = _c2f_inputs(lens, seed=601, clustered=True)
    q, kv = syn.mla_attention(2, inp.key_pool.shape[0], seed=602)
    wl = W.build("c2f", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)), c2f=True)
    full = W.build("full", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)))
    wl.step()
    full.step()
    torch.cuda.synchronize()
    assert_status_clean()
    assert torch.equal(wl.idx, full.idx)
    assert torch.equal(wl.o, full.o)
    n = wl.tensors["n_survivors"].cpu().numpy()
    assert (n < np.array([-(-L // 64) for L in lens]) * 0.5).all()
    _check_mla_step(full, inp, q, kv, 2048, heads_sample=slice(0, 128, 16))
    # the same step with the original keys in pinned host memory (small staging: several
    # passes over the survivors): the same selection and output
    host = W.build("c2f_host", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)), c2f=True,
                   c2f_keys_on_host=True, c2f_stage_blocks=64)
    host.step()
    torch.cuda.synchronize()
    assert_status_clean()
    assert torch.equal(host.idx, full.idx)
    assert torch.equal(host.o, full.o)
    assert torch.equal(host.tensors["n_survivors"], wl.tensors["n_survivors"])


@pytest.mark.parametrize("lens", [[20000, 9000], [16384] * 8])
def test_decode_step_writes_outputs_to_host_memory(lens):
    """o and lse are plain addresses: with pinned host buffers the step's last kernel writes
    them over the host link, and the bits equal those of the step with device outputs (two
    requests: 16 KV splits; eight: the per-request completion counts)."""
    inp = syn.indexer_fp8(lens, seed=701)
    q, kv = syn.mla_attention(len(lens), inp.key_pool.shape[0], seed=702)
    wl = W.build("host_out", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)))
    wl.step()
    torch.cuda.synchronize()
    ref_o, ref_lse = wl.o.cpu(), wl.lse.cpu()
    host_o = torch.full(ref_o.shape, float("nan"), dtype=ref_o.dtype).pin_memory()
    host_lse = torch.full(ref_lse.shape, float("nan")).pin_memory()
    dev_o, dev_lse = wl.args.attn.o, wl.args.attn.lse
    wl.args.attn.o, wl.args.attn.lse = host_o.data_ptr(), host_lse.data_ptr()
    for _ in range(2):  # twice: the per-request counts start from zero again every step
        wl.step()
        torch.cuda.synchronize()
        assert torch.equal(host_o, ref_o) and torch.equal(host_lse, ref_lse)
    wl.args.attn.o, wl.args.attn.lse = dev_o, dev_lse
    assert_status_clean()


@pytest.mark.parametrize("kind", ["iid", "ties_at_k", "all_equal", "clustered", "ragged"])
def test_decode_step_selection_equals_full_topk(kind):
    """The step's selection (indexer candidates + candidate top-k, or the cluster top-k where
    the candidates do not serve) equals ls_topk_select over the same scores bit for bit --
    positions and selection scores -- for scores drawn i.i.d., for 600 tokens given the key of
    the token ranked ~2000th (exact ties across the k-th score: the lower positions must win),
    for scores that all tie (too many equal keys: the cluster top-k decides), for
    block-clustered keys (a skewed request), and for a ragged batch whose short requests give
    fewer candidates than k or leave indexer CTAs without tiles (those go to the cluster
    top-k, the long one to the candidates)."""
    lens = [131072, 3000, 40000, 1] if kind == "ragged" else [131072, 131072, 100000, 70001]
    if kind == "clustered":
        from test_gpu_stages import _c2f_inputs
        inp = _c2f_inputs(lens, seed=801, clustered=True)
    else:
        inp = syn.indexer_fp8(lens, seed=801)
        if kind == "all_equal":
            inp.key_pool[:] = inp.key_pool[0, 0]
            inp.key_scale[:] = inp.key_scale[0, 0]
        elif kind == "ties_at_k":
            sc = gpu_index_scores(inp).cpu()
            g = torch.Generator().manual_seed(803)
            pt = inp.page_table
            for b, L in enumerate(lens):
                src = int(torch.argsort(sc[b, :L], descending=True)[2000])
                dst = torch.randperm(L, generator=g)[:600]
                sp, so = int(pt[b, src // 64]), src % 64
                for d in dst.tolist():
                    inp.key_pool[int(pt[b, d // 64]), d % 64] = inp.key_pool[sp, so]
                    inp.key_scale[int(pt[b, d // 64]), d % 64] = inp.key_scale[sp, so]
    q, kv = syn.mla_attention(len(lens), inp.key_pool.shape[0], seed=802)
    wl = W.build("cand", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)))
    for _ in range(2):  # the filter's counts restart every step
        wl.step()
        torch.cuda.synchronize()
        assert_status_clean()
        scores = gpu_index_scores_from(wl)
        full = torch.full_like(wl.idx, -7)
        full_sel = torch.zeros_like(wl.tensors["sel"])
        B.ls_topk_select(scores=scores, lens=wl.tensors["i_lens"], idx=full, sel_score=full_sel)
        torch.cuda.synchronize()
        assert torch.equal(wl.idx, full)
        assert torch.equal(wl.tensors["sel"], full_sel)


def gpu_index_scores_from(wl):
    """The indexer's scores for the workload's own device inputs."""
    t = wl.tensors
    scores = torch.full((wl.batch, wl.args.index.max_len), float("nan"), device=DEV)
    B.ls_index_score(q=t["i_q"], w=t["i_w"], key_pool=t["i_key_pool"], page_table=t["i_page_table"],
                     lens=t["i_lens"], scores=scores, q_scale=t["i_q_scale"], key_scale=t["i_key_scale"])
    return scores
