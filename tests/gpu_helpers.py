"""Shared helpers of the GPU parity tests: move synthetic inputs to the device, call
the C ABI through the binding, and convert inputs for the oracle."""
import numpy as np
import torch

from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import synthetic as syn

DEV = "cuda"


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (oracle input)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_index_inputs(inp: syn.IndexerInputs):
    if inp.key_format == "e4m3":
        return dict(q=inp.q.numpy(), w=bits16(inp.w), key_pool=inp.key_pool.numpy(),
                    page_table=inp.page_table.numpy(), lens=inp.lens.tolist(), q_scale=inp.q_scale.numpy(),
                    key_scale_pool=inp.key_scale.numpy())
    return dict(q=inp.q.numpy(), w=inp.w.numpy(), key_pool=inp.key_pool.numpy(), page_table=inp.page_table.numpy(),
                lens=inp.lens.tolist(), key_format="f32", w_format="f32")


def to_dev(inp: syn.IndexerInputs):
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.__dict__.items() if k != "extra"}
    return d


def round4(x):
    return (int(x) + 3) // 4 * 4


def gpu_index_scores(inp: syn.IndexerInputs, variant=0, max_len=None):
    d = to_dev(inp)
    ml = round4(max_len or inp.max_len)
    scores = torch.full((inp.batch, ml), float("nan"), device=DEV)
    B.ls_index_score(q=d["q"], w=d["w"], key_pool=d["key_pool"], page_table=d["page_table"], lens=d["lens"],
                     scores=scores, q_scale=d["q_scale"], key_scale=d["key_scale"], variant=variant)
    torch.cuda.synchronize()
    return scores


def assert_status_clean():
    flags = B.ls_check_device_status()
    assert flags == 0, f"device status bits 0x{flags:x}"


def check_topk_band(gpu_idx_row, oracle_scores_row, k, rel=1e-3):
    """Top-k index sets equal except for positions whose oracle score lies within
    `rel` (relative) of the oracle's k-th score; equal cardinality; ascending order."""
    import oracle.ls_oracle as O
    s = np.asarray(oracle_scores_row, dtype=np.float64)
    L = s.shape[0]
    ref, _ = O.topk_select(s, k)
    g = np.asarray(gpu_idx_row)
    n = min(k, L)
    assert (g[n:] == -1).all(), "padding must be -1"
    gv = g[:n]
    assert (np.diff(gv) > 0).all(), "indices must be strictly ascending"
    assert gv.min() >= 0 and gv.max() < L
    diff = set(gv.tolist()) ^ set(ref[:n].tolist())
    if diff:
        tau = np.sort(s)[::-1][n - 1]
        bad = [p for p in diff if abs(s[p] - tau) > rel * abs(tau)]
        assert not bad, f"{len(bad)} positions outside the tie band, e.g. {bad[:5]}"
    return len(diff)
