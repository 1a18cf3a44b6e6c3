"""Pins for the CPU oracle: every check here ties the oracle to something other than
itself (a spec table, a library routine, a hand-worked example, a closed form, an
invariant, or brute force on a tiny input).  CPU only."""
import math
import os

import numpy as np
import pytest
import torch

import oracle.ls_oracle as O
from sparse_attention_decode_ls_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- formats
def _known_e4m3():
    out = []
    with open(os.path.join(GOLDEN, "e4m3_known_values.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            code, val = line.split()
            out.append((int(code, 16), float(val)))
    return out


def test_e4m3_spec_values():
    tab = O.e4m3_values()
    for code, val in _known_e4m3():
        if math.isnan(val):
            assert math.isnan(tab[code])
        else:
            assert tab[code] == val and math.copysign(1, tab[code]) == math.copysign(1, val), hex(code)


def test_e4m3_matches_torch_all_codes():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    tab = O.e4m3_values()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(tab))
    assert np.array_equal(ref[~nan], tab[~nan])


def test_bf16_decode_matches_torch():
    bits = torch.arange(0, 65536, 7, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).double().numpy()
    got = O.bf16_decode(bits.numpy().view(np.uint16))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_directed_rounding_brute_force():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 2000), rng.uniform(-1, 1, 2000),
                        O.e4m3_values()[np.isfinite(O.e4m3_values())]])
    finite = np.array(sorted(set(v for v in O.e4m3_values() if np.isfinite(v))))
    up = O.e4m3_decode(O.f32_round_up_to_e4m3_code(x))
    dn = O.e4m3_decode(O.f32_round_down_to_e4m3_code(x))
    for xi, u, d in zip(x, up, dn):
        assert u == min(v for v in finite if v >= xi)
        assert d == max(v for v in finite if v <= xi)


# ----------------------------------------------------------------------------- indexer
def _hand_indexer():
    q8 = np.array([[[0x38, 0xC0], [0x40, 0x30]]], dtype=np.uint8)
    sq = np.array([[0.5, 1.0]], dtype=np.float32)
    w = np.array([[0x3F80, 0xBF00]], dtype=np.uint16)
    pool = np.zeros((1, 64, 2), dtype=np.uint8)
    pool[0, :3] = [[0x38, 0x38], [0x40, 0xB8], [0xB8, 0x30]]
    ks = np.ones((1, 64), dtype=np.float32)
    ks[0, :3] = [2.0, 1.0, 4.0]
    pt = np.zeros((1, 1), dtype=np.int32)
    return q8, sq, w, pool, ks, pt


def test_index_score_hand_example():
    q8, sq, w, pool, ks, pt = _hand_indexer()
    s = O.index_score(q8, w, pool, pt, [3], q_scale=sq, key_scale_pool=ks)
    assert np.array_equal(s[0], [-2.5, 0.25, 0.0])


def test_topk_hand_example():
    s = np.array([-2.5, 0.25, 0.0])
    idx, sel = O.topk_select(s, 2)
    assert idx.tolist() == [1, 2] and sel.tolist() == [0.25, 0.0]
    idx, _ = O.topk_select(s, 4)
    assert idx.tolist() == [0, 1, 2, -1]


def test_decode_step_hand_example():
    """The composed step on the hand example (tests/golden/hand_examples.md, decode step):
    the indexer's top 2 are positions 1 and 2, and one head over their rows gives closed forms."""
    q8, sq, w, pool, ks, pt = _hand_indexer()
    kv = np.zeros((1, 64, 2), dtype=np.uint16)
    kv[0, :3] = [[0x4040, 0x4110], [0x3F80, 0x4000], [0x0000, 0x4080]]
    q_attn = np.array([[[0x3F80, 0x0000]]], dtype=np.uint16)
    scores, idx, o, lse = O.decode_step(q8=q8, q_scale=sq, w_bits=w, key_pool=pool, key_scale_pool=ks,
                                        page_table=pt, lens=[3], k=2, q_attn_bits=q_attn, kv_pool_bits=kv,
                                        scale=1.0, dv=1)
    assert np.array_equal(np.asarray(scores[0])[:3], [-2.5, 0.25, 0.0])
    assert idx.tolist() == [[1, 2]]
    e = math.e
    assert o.shape == (1, 1, 1) and abs(o[0, 0, 0] - e / (1 + e)) < 1e-15
    assert abs(lse[0, 0] - math.log1p(e)) < 1e-15


def test_index_score_page_shuffle_invariance():
    inp = syn.indexer_fp8([700, 300], heads=8, dim=32, seed=5)
    a = O.index_score(inp.q.numpy(), inp.w.view(torch.int16).numpy().view(np.uint16),
                      inp.key_pool.numpy(), inp.page_table.numpy(), inp.lens.tolist(),
                      q_scale=inp.q_scale.numpy(), key_scale_pool=inp.key_scale.numpy())
    # move every physical page somewhere else and fix up the page table
    n = inp.key_pool.shape[0]
    perm = np.random.default_rng(1).permutation(n)
    pool2 = np.empty_like(inp.key_pool.numpy())
    ks2 = np.empty_like(inp.key_scale.numpy())
    pool2[perm] = inp.key_pool.numpy()
    ks2[perm] = inp.key_scale.numpy()
    pt2 = perm[inp.page_table.numpy()].astype(np.int32)
    b = O.index_score(inp.q.numpy(), inp.w.view(torch.int16).numpy().view(np.uint16), pool2, pt2,
                      inp.lens.tolist(), q_scale=inp.q_scale.numpy(), key_scale_pool=ks2)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_index_score_single_head_closed_form():
    # one head, w = 1: the score is ReLU of the dequantised dot product
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 16)).astype(np.float32)
    keys = rng.standard_normal((1, 64, 16)).astype(np.float32)
    s = O.index_score(q, np.ones((1, 1), np.float32), keys, np.zeros((1, 1), np.int32), [64],
                      key_format="f32", w_format="f32")[0]
    dots = np.array([sum(float(q[0, 0, d]) * float(keys[0, t, d]) for d in range(16)) for t in range(64)])
    assert np.allclose(s, np.maximum(dots, 0.0), rtol=1e-12, atol=1e-12)
    assert (s[dots < 0] == 0).all()


# ----------------------------------------------------------------------------- top-k
def test_topk_vs_python_sorted_with_ties():
    rng = np.random.default_rng(3)
    for trial in range(200):
        L = int(rng.integers(1, 60))
        k = int(rng.integers(1, 70))
        s = rng.integers(-3, 4, size=L).astype(np.float64)  # many ties
        ref = sorted(range(L), key=lambda i: (-s[i], i))[:k]
        idx, sel = O.topk_select(s, k)
        exp = sorted(ref) + [-1] * max(0, k - L)
        assert idx.tolist() == exp


def test_topk_permutation_identity():
    rng = np.random.default_rng(4)
    s = rng.standard_normal(5000)
    perm = rng.permutation(5000)
    a, _ = O.topk_select(s, 300)
    b, _ = O.topk_select(s[perm], 300)
    # position i of the permuted history holds token perm[i]
    assert sorted(perm[b].tolist()) == a.tolist()


# ----------------------------------------------------------------------------- attention
def test_attention_equals_full_attention_when_k_covers_history():
    rng = np.random.default_rng(5)
    H, L, D, Dv = 8, 50, 32, 24
    q = rng.standard_normal((H, D))
    kv = rng.standard_normal((L, D))
    scale = 1 / math.sqrt(D)
    o, lse = O.sparse_attn_decode(q, kv, kv[:, :Dv], scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(kv)[None, None].expand(1, H, L, D),
        torch.from_numpy(kv[:, :Dv])[None, None].expand(1, H, L, Dv), scale=scale)[0, :, 0]
    assert np.allclose(o, ref.numpy(), rtol=1e-12, atol=1e-12)
    ref_lse = torch.logsumexp(scale * torch.from_numpy(q) @ torch.from_numpy(kv).T, dim=1).numpy()
    assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_uniform_closed_form():
    rng = np.random.default_rng(6)
    n, D = 37, 16
    krow = rng.standard_normal(D)
    K = np.tile(krow, (n, 1))
    V = rng.standard_normal((n, D))
    q = rng.standard_normal((3, D))
    o, lse = O.sparse_attn_decode(q, K, V, 0.25)
    assert np.allclose(o, V.mean(0)[None].repeat(3, 0), atol=1e-12)
    assert np.allclose(lse, 0.25 * (q @ krow) + math.log(n), atol=1e-12)


def test_attention_single_row_and_empty():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((2, 8))
    K = rng.standard_normal((1, 8))
    o, lse = O.sparse_attn_decode(q, K, K, 0.5)
    assert np.allclose(o, np.repeat(K, 2, 0)) and np.allclose(lse, 0.5 * (q @ K[0]))
    o, lse = O.sparse_attn_decode(q, K[:0], K[:0], 0.5)
    assert (o == 0).all() and np.isneginf(lse).all()


def test_selected_rows_through_page_table():
    pool = np.arange(3 * 64 * 2).reshape(3, 64, 2)
    pt = np.array([2, 0, 1])
    rows = O.selected_rows(pool, pt, [0, 65, 130, -1])
    assert rows.tolist() == [pool[2, 0].tolist(), pool[0, 1].tolist(), pool[1, 2].tolist()]


# ----------------------------------------------------------------------------- coarse-to-fine
def test_block_summary_hand_example():
    pool = np.zeros((1, 64, 2), dtype=np.uint8)
    pool[0, 0] = [0x5E, 0xD6]
    pool[0, 1] = [0x52, 0x44]
    ks = np.ones((1, 64), dtype=np.float32)
    kmax8, kmin8, bs = O.block_summaries(pool, ks, np.array([0]), 2)
    assert kmax8.tolist() == [[0x7E, 0x64]] and kmin8.tolist() == [[0x72, 0xF6]]
    assert bs.tolist() == [0.0625]


def _random_c2f_case(seed, clustered, L=64 * 40 + 17, H=16, D=32, w_nonneg=True):
    if clustered:
        g = torch.Generator().manual_seed(seed)
        qf = torch.randn((1, H, D), generator=g)
        nb = -(-L // 64)
        keys = syn.clustered_keys(nb, 1, dim=D, within_sigma=0.05, shift_frac=0.1,
                                  direction=qf.sum(1), seed=seed)[:L]
        inp = syn.indexer_fp8([L], heads=H, dim=D, seed=seed, w_nonneg=w_nonneg, q=qf,
                              keys=syn.logical_to_pool(keys, [L], syn.page_layout([L], seed + 17)[0],
                                                       nb))
    else:
        inp = syn.indexer_fp8([L], heads=H, dim=D, seed=seed, w_nonneg=w_nonneg)
    return inp


@pytest.mark.parametrize("seed,clustered,w_nonneg", [(11, False, True), (12, True, True),
                                                      (13, True, False), (14, False, False)])
def test_block_bound_dominates_block_scores(seed, clustered, w_nonneg):
    inp = _random_c2f_case(seed, clustered, w_nonneg=w_nonneg)
    L = int(inp.lens[0])
    wb = inp.w.view(torch.int16).numpy().view(np.uint16)
    s = O.index_score(inp.q.numpy(), wb, inp.key_pool.numpy(), inp.page_table.numpy(), [L],
                      q_scale=inp.q_scale.numpy(), key_scale_pool=inp.key_scale.numpy())[0]
    kmax8, kmin8, bs = O.block_summaries(inp.key_pool.numpy(), inp.key_scale.numpy(),
                                         inp.page_table.numpy()[0], L)
    # the stored box contains every dequantised key (outward rounding)
    k8 = O._rows_of_request(inp.key_pool.numpy(), inp.page_table.numpy()[0], L)
    kk = O._rows_of_request(inp.key_scale.numpy(), inp.page_table.numpy()[0], L)
    keys = O.e4m3_decode(k8) * kk.astype(np.float64)[:, None]
    Kmax = O.e4m3_decode(kmax8) * bs[:, None]
    Kmin = O.e4m3_decode(kmin8) * bs[:, None]
    for j in range(kmax8.shape[0]):
        blk = keys[j * 64:(j + 1) * 64]
        assert (Kmax[j] >= blk.max(0)).all() and (Kmin[j] <= blk.min(0)).all()
    ub = O.block_bound(inp.q.numpy()[0], inp.q_scale.numpy()[0], wb[0], kmax8, kmin8, bs)
    for j in range(ub.shape[0]):
        assert ub[j] >= s[j * 64:(j + 1) * 64].max() - 1e-9 * abs(ub[j])


def test_block_bound_is_tight_for_constant_block():
    # all tokens of the block equal and exactly representable: the box collapses to
    # the key itself, so the bound equals the score exactly (any sign of w)
    H, D = 4, 8
    rng = np.random.default_rng(9)
    q8 = rng.choice([0x38, 0xB8, 0x40, 0xC0, 0x30, 0x00], size=(1, H, D)).astype(np.uint8)
    sq = np.array([[1.0, 0.5, 2.0, 1.0]], np.float32)
    w = np.array([[0x3F80, 0xBF00, 0x3F00, 0xC000]], np.uint16)  # 1, -0.5, 0.5, -2
    # key values from {7, 3.5, -1.75, 1, -2, 0.5, -7} with amax 7: the block scale is
    # 7/448 = 2^-6 and every key / scale is an e4m3 value, so the box is exact
    code = rng.choice([0x4E, 0x46, 0xBE, 0x38, 0xC0, 0x30, 0xCE], size=D).astype(np.uint8)
    code[0] = 0x4E
    pool = np.tile(code, (1, 64, 1))
    ks = np.ones((1, 64), np.float32)
    s = O.index_score(q8, w, pool, np.zeros((1, 1), np.int32), [64], q_scale=sq, key_scale_pool=ks)[0]
    kmax8, kmin8, bs = O.block_summaries(pool, ks, np.array([0]), 64)
    ub = O.block_bound(q8[0], sq[0], w[0], kmax8, kmin8, bs)
    assert bs[0] == 2.0 ** -6 and (kmax8 == kmin8).all()
    assert np.allclose(ub[0], s[0], rtol=1e-12) and np.allclose(s, s[0])


@pytest.mark.parametrize("seed,clustered,k", [(21, True, 128), (22, False, 128), (23, True, 300),
                                               (24, True, 64 * 50)])
def test_c2f_equals_full_scan(seed, clustered, k):
    inp = _random_c2f_case(seed, clustered)
    L = int(inp.lens[0])
    wb = inp.w.view(torch.int16).numpy().view(np.uint16)
    s = O.index_score(inp.q.numpy(), wb, inp.key_pool.numpy(), inp.page_table.numpy(), [L],
                      q_scale=inp.q_scale.numpy(), key_scale_pool=inp.key_scale.numpy())[0]
    kmax8, kmin8, bs = O.block_summaries(inp.key_pool.numpy(), inp.key_scale.numpy(),
                                         inp.page_table.numpy()[0], L)
    ub = O.block_bound(inp.q.numpy()[0], inp.q_scale.numpy()[0], wb[0], kmax8, kmin8, bs)
    tau0, surv, idx, _ = O.c2f_prune(s, ub, k)
    full, _ = O.topk_select(s, k)
    assert idx.tolist() == full.tolist()
    # every block holding a selected token survives
    assert set((full[full >= 0] // 64).tolist()) <= set(surv.tolist())
    if clustered and k <= 300:
        assert surv.size < ub.size  # clustered keys do prune


# ----------------------------------------------------------------------------- hot buffer
def test_hotbuf_hand_example():
    r = O.hotbuf_resolve([2, 4, 8], [1.5, 2.5, 3.5], [5, -1, 2, 7], [0.9, 0.0, 0.1, 0.5],
                         [-1, -1, 2, -1, -1, 0, -1, 3, -1, -1])
    assert r["sel_slot"].tolist() == [2, 1, 3]
    assert r["miss_pos"].tolist() == [4, 8, -1] and r["miss_slot"].tolist() == [1, 3, -1]
    assert r["n_miss"] == 2
    assert r["pos_of_slot"].tolist() == [5, 4, 2, 8]
    assert r["slot_of_pos"].tolist() == [-1, -1, 2, -1, 1, 0, -1, -1, 3, -1]
    assert np.allclose(r["recent_score"], [0.9, 2.5, 1.5, 3.5])


@pytest.mark.parametrize("seed", range(6))
def test_hotbuf_invariants_and_brute_force(seed):
    rng = np.random.default_rng(seed)
    S, L, k = 16, 60, int(rng.integers(1, 12))
    resident = rng.choice(L, size=int(rng.integers(0, S + 1)), replace=False)
    slots = rng.choice(S, size=resident.size, replace=False)
    pos_of_slot = np.full(S, -1, np.int32)
    slot_of_pos = np.full(L, -1, np.int32)
    pos_of_slot[slots] = resident
    slot_of_pos[resident] = slots
    recent = rng.integers(0, 4, S).astype(np.float32)  # ties on purpose
    sel = np.sort(rng.choice(L, size=k, replace=False)).astype(np.int32)
    sc = rng.standard_normal(k).astype(np.float32)
    r = O.hotbuf_resolve(sel, sc, pos_of_slot, recent, slot_of_pos)
    hits = [p for p in sel if slot_of_pos[p] >= 0]
    misses = [p for p in sel if slot_of_pos[p] < 0]
    assert r["n_miss"] == len(misses) and r["miss_pos"][:len(misses)].tolist() == misses
    pinned = {int(slot_of_pos[p]) for p in hits}
    victims = r["miss_slot"][: len(misses)].tolist()
    assert not (set(victims) & pinned) and len(set(victims)) == len(victims)
    # brute force: no unpinned non-victim slot precedes a victim in (empty, score, slot) order
    key = lambda s: (0, 0.0, s) if pos_of_slot[s] < 0 else (1, float(recent[s]), s)
    others = [s for s in range(S) if s not in pinned and s not in victims]
    for v in victims:
        assert all(key(v) < key(o) for o in others)
    assert [key(v) for v in victims] == sorted(key(v) for v in victims)
    # maps are inverse and every selected position is resident afterwards
    P, Q = r["pos_of_slot"], r["slot_of_pos"]
    for s in range(S):
        if P[s] >= 0:
            assert Q[P[s]] == s
    for p in range(L):
        if Q[p] >= 0:
            assert P[Q[p]] == p
    for j, p in enumerate(sel):
        assert Q[p] == r["sel_slot"][j] >= 0
        assert r["recent_score"][Q[p]] == sc[j]


def test_gather_is_a_byte_copy():
    rng = np.random.default_rng(8)
    host = rng.integers(0, 255, size=(4, 64, 16), dtype=np.uint8)
    pt = np.array([3, 1])
    hbuf = rng.integers(0, 255, size=(8, 16), dtype=np.uint8)
    out = O.gather_misses(host, pt, [5, 70], [6, 2], 2, hbuf)
    assert np.array_equal(out[6], host[3, 5]) and np.array_equal(out[2], host[1, 6])
    keep = [0, 1, 3, 4, 5, 7]
    assert np.array_equal(out[keep], hbuf[keep])


# ----------------------------------------------------------------------------- planted mistakes
def test_planted_mistakes_are_caught(monkeypatch):
    """Break the oracle on purpose (CPU only) and check that a pin above fails."""
    q8, sq, w, pool, ks, pt = _hand_indexer()
    # dropped ReLU
    real_max = np.maximum
    monkeypatch.setattr(O.np, "maximum", lambda a, b, *x, **kw: a if (np.isscalar(b) and b == 0.0)
                        else real_max(a, b, *x, **kw))
    s = O.index_score(q8, w, pool, pt, [3], q_scale=sq, key_scale_pool=ks)[0]
    assert not np.array_equal(s, [-2.5, 0.25, 0.0])
    monkeypatch.undo()
    # e4m3 exponent bias off by one
    bad = O.e4m3_values() * 2.0
    monkeypatch.setattr(O, "_E4M3", bad)
    s = O.index_score(q8, w, pool, pt, [3], q_scale=sq, key_scale_pool=ks)[0]
    assert not np.array_equal(s, [-2.5, 0.25, 0.0])
    monkeypatch.undo()
    # transposed tie rule (higher position first) breaks the brute-force top-k pin
    s = np.array([1.0, 1.0, 0.0])
    idx, _ = O.topk_select(s, 1)
    assert idx.tolist() == [0]
