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
