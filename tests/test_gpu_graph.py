"""ls_decode_step can be captured in a CUDA graph (no allocation, no host sync inside)
and the replay reproduces the eager step bit for bit."""
import pytest
import torch

from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import synthetic as syn
from sparse_attention_decode_ls_b200 import workload as W

pytestmark = pytest.mark.gpu


def test_decode_step_graph_replay_matches_eager():
    lens = [30000, 17000, 64 * 200]
    inp = syn.indexer_fp8(lens, seed=901)
    q, kv = syn.mla_attention(len(lens), inp.key_pool.shape[0], seed=902)
    wl = W.build("graph", inp, k=2048, attn=dict(q=q, kv=kv, scale=syn.softmax_scale(576)))
    wl.step()
    torch.cuda.synchronize()
    o_ref, lse_ref, idx_ref = wl.o.clone(), wl.lse.clone(), wl.idx.clone()
    wl.o.zero_()
    wl.idx.fill_(-5)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        wl.step()  # warm up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        wl.step()
    for _ in range(3):
        wl.o.zero_()
        wl.idx.fill_(-5)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(wl.idx, idx_ref)
        assert torch.equal(wl.o, o_ref)
        assert torch.equal(wl.lse, lse_ref)
    assert B.ls_check_device_status() == 0


def test_hot_buffer_step_graph_replay_matches_eager():
    """The hot-buffer step forks the resident-row attention onto a second stream while the
    misses are copied in from pinned host memory; the fork and join are captured too."""
    lens = [40000, 64 * 300 + 5]
    inp = syn.indexer_fp8(lens, seed=911)
    n_pool = inp.key_pool.shape[0]
    q, kv = syn.mla_attention(len(lens), n_pool, seed=912)
    host = kv.view(torch.int16).pin_memory().view(torch.bfloat16)
    ml = (max(lens) + 3) // 4 * 4
    # a buffer that holds a seeded half of some other positions: most of the selection misses
    g0 = torch.Generator().manual_seed(913)
    other = [torch.randperm(L, generator=g0)[:1024] for L in lens]
    pos_of_slot, slot_of_pos, recent = syn.hot_buffer_state(other, lens, n_slots=4096, miss_frac=0.5, seed=914,
                                                            max_len=ml)
    wl = W.build("graph_hotbuf", inp, k=2048, attn=dict(q=q, kv_host=True, scale=syn.softmax_scale(576)),
                 hotbuf=dict(pos_of_slot=pos_of_slot, slot_of_pos=slot_of_pos, recent=recent, host_kv=host))
    state = ("pos_of_slot", "slot_of_pos", "hbuf", "n_miss")
    wl.restore_hotbuf()
    wl.step()
    torch.cuda.synchronize()
    ref = {key: wl.tensors[key].clone() for key in ("o", "lse", "idx") + state}
    assert int(ref["n_miss"].min()) > 0
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        wl.restore_hotbuf()
        wl.step()  # warm up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        wl.step()
    for _ in range(3):
        wl.restore_hotbuf()
        wl.o.zero_()
        wl.idx.fill_(-5)
        wl.tensors["n_miss"].fill_(-1)
        g.replay()
        torch.cuda.synchronize()
        for key, val in ref.items():
            assert torch.equal(wl.tensors[key], val), key
    assert B.ls_check_device_status() == 0


def test_full_size_step_is_deterministic():
    """Race check without a sanitizer: the full-size step (batch 8 at 131,072 tokens), run
    three times on the same inputs with L2 evicted in between, gives bit-identical selection,
    output and log-sum-exp."""
    wl = W.mla_decode(batch=8, ctx=131072, k=2048, seed=1002, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        flush.zero_()
        wl.o.zero_()
        wl.idx.fill_(-5)
        wl.step()
        torch.cuda.synchronize()
        outs.append((wl.idx.clone(), wl.o.clone(), wl.lse.clone()))
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)
    assert B.ls_check_device_status() == 0
