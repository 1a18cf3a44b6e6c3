"""Layer-streaming prefill (LeanSparse, abstract: each layer's history streams through two
reusable GPU buffers): per-layer block summaries built from staged copies of the host
history, and hot buffers seeded with each request's most recent positions."""
import numpy as np
import pytest
import torch

import oracle.ls_oracle as O
from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import synthetic as syn

from gpu_helpers import DEV, assert_status_clean, round4

pytestmark = pytest.mark.gpu


def _layers(lens, n_layers, seed):
    table, n_pool = syn.page_layout(lens, seed)
    g = torch.Generator().manual_seed(seed + 1)
    keys, scales, kv = [], [], []
    for _ in range(n_layers):
        k8, sk = syn.quantize_e4m3(torch.randn((n_pool * 64, 128), generator=g))
        keys.append(k8.view(n_pool, 64, 128).pin_memory())
        scales.append(sk.view(n_pool, 64).contiguous().pin_memory())
        kv.append(torch.randn((n_pool, 64, 576), generator=g).to(torch.bfloat16).view(torch.int16).pin_memory())
    return table, n_pool, keys, scales, kv


@pytest.mark.parametrize("n_slots", [0, 4096])
def test_prefill_stream_summaries_and_seed(n_slots):
    lens = [64 * 300 + 17, 64 * 41, 5000]
    n_layers = 3
    table, n_pool, keys, scales, kv = _layers(lens, n_layers, seed=71)
    Bn, ml = len(lens), round4(max(lens))
    mb = max(-(-L // 64) for L in lens)
    summ = [torch.zeros((Bn, mb, 256), dtype=torch.uint8, device=DEV) for _ in range(n_layers)]
    bsc = [torch.zeros((Bn, mb), device=DEV) for _ in range(n_layers)]
    seed = {}
    if n_slots:
        seed = dict(host_kv=kv,
                    hbuf=[torch.full((Bn, n_slots, 576), 7, dtype=torch.int16, device=DEV) for _ in range(n_layers)],
                    pos_of_slot=[torch.full((Bn, n_slots), -5, dtype=torch.int32, device=DEV) for _ in range(n_layers)],
                    slot_of_pos=[torch.full((Bn, ml), -5, dtype=torch.int32, device=DEV) for _ in range(n_layers)],
                    recent_score=[torch.full((Bn, n_slots), 3.0, device=DEV) for _ in range(n_layers)])
    a = B.prefill_args(page_table=table.to(DEV), lens=torch.tensor(lens, dtype=torch.int32, device=DEV), max_len=ml,
                       host_keys=keys, host_key_scales=scales, summaries=summ, block_scale=bsc, **seed)
    ws = torch.empty(B.ls_prefill_stream_workspace_size(a), dtype=torch.uint8, device=DEV)
    B.ls_prefill_stream(a, ws)
    torch.cuda.synchronize()
    assert_status_clean()
    tb = table.numpy()
    for layer in range(n_layers):
        for b, L in enumerate(lens):
            kmax8, kmin8, bs = O.block_summaries(keys[layer].numpy(), scales[layer].numpy(), tb[b], L)
            nb = kmax8.shape[0]
            assert np.array_equal(summ[layer][b, :nb, :128].cpu().numpy(), kmax8)
            assert np.array_equal(summ[layer][b, :nb, 128:].cpu().numpy(), kmin8)
            assert np.array_equal(bsc[layer][b, :nb].cpu().numpy(), bs)
            if not n_slots:
                continue
            first = L - n_slots
            want_pos = np.array([first + s if first + s >= 0 else -1 for s in range(n_slots)])
            assert np.array_equal(seed["pos_of_slot"][layer][b].cpu().numpy(), want_pos)
            want_sop = np.full(ml, -1)
            for s, p in enumerate(want_pos):
                if p >= 0:
                    want_sop[p] = s
            assert np.array_equal(seed["slot_of_pos"][layer][b].cpu().numpy(), want_sop)
            assert (seed["recent_score"][layer][b] == 0).all()
            hb = seed["hbuf"][layer][b].cpu().numpy()
            hist = kv[layer].numpy()
            for s, p in enumerate(want_pos):
                if p >= 0:
                    assert np.array_equal(hb[s], hist[tb[b, p // 64], p % 64])
                else:
                    assert (hb[s] == 7).all()  # an empty slot's row is left as it was


def test_prefill_rejects_pageable_host_keys():
    lens = [64 * 10]
    table, n_pool, keys, scales, _ = _layers(lens, 1, seed=72)
    summ = [torch.zeros((1, 10, 256), dtype=torch.uint8, device=DEV)]
    bsc = [torch.zeros((1, 10), device=DEV)]
    a = B.prefill_args(page_table=table.to(DEV), lens=torch.tensor(lens, dtype=torch.int32, device=DEV), max_len=640,
                       host_keys=[keys[0].clone()], host_key_scales=scales, summaries=summ, block_scale=bsc)
    ws = torch.empty(B.ls_prefill_stream_workspace_size(a), dtype=torch.uint8, device=DEV)
    with pytest.raises(B.LsError, match="pinned"):
        B.ls_prefill_stream(a, ws)
