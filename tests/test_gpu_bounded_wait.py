"""A wait inside a kernel that nothing completes gives up after the wait limit, raises
LS_DEV_TIMEOUT and returns: the context stays usable (no trap, no hang)."""
import time

import pytest
import torch

from sparse_attention_decode_ls_b200 import binding as B

from gpu_helpers import DEV, assert_status_clean

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    assert_status_clean()
    B.ls_set_wait_limit(2_000_000)  # 2 ms
    try:
        t0 = time.perf_counter()
        B.ls_selftest_bounded_wait()
        flags = B.ls_check_device_status()
        elapsed = time.perf_counter() - t0
    finally:
        B.ls_set_wait_limit(2_000_000_000)
    assert flags & B.LS_DEV_TIMEOUT
    assert elapsed < 1.0
    # the context still runs work afterwards
    s = torch.randn((1, 4096), device=DEV)
    idx = torch.empty((1, 64), dtype=torch.int32, device=DEV)
    B.ls_topk_select(scores=s, lens=torch.tensor([4096], dtype=torch.int32, device=DEV), idx=idx)
    torch.cuda.synchronize()
    assert torch.equal(idx.cpu(), torch.topk(s.cpu(), 64).indices.sort().values.int())
    assert_status_clean()


def test_wait_limit_range_is_checked():
    with pytest.raises(B.LsError):
        B.ls_set_wait_limit(10)
