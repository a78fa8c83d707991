"""The device's bounded waits: a wait on an mbarrier that no copy completes
gives up after the kernels' limit, reports LOOPKV_DEVERR_TIMEOUT through the
error word, and the context stays usable (a decode runs right after)."""

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_wait_gives_up_and_reports_timeout():
    from mixed_precision_kv_loopkv_b200 import (LOOPKV_DEVERR_TIMEOUT, KVCells, loopkv_decode_attention,
                                                loopkv_quantize_append, loopkv_selftest_wait_timeout)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    loopkv_selftest_wait_timeout(err, elapsed)
    torch.cuda.synchronize()
    assert int(err) == LOOPKV_DEVERR_TIMEOUT
    assert 2.0e9 <= int(elapsed) < 6.0e9
    # the context still runs kernels: a small append + decode
    kv = KVCells(["q4"], 1, 1, 1, 64, 4, 1, 4)
    k = torch.randn(1, 40, 1, 64, device="cuda").to(torch.bfloat16)
    table = torch.arange(4, dtype=torch.int32, device="cuda").view(1, 4)
    loopkv_quantize_append(kv, 0, 0, k, k.clone(), table, torch.zeros(1, dtype=torch.int32, device="cuda"))
    out = loopkv_decode_attention(kv, 0, 0, torch.randn(1, 1, 64, device="cuda").to(torch.bfloat16), table,
                                  torch.tensor([40], dtype=torch.int32, device="cuda"), 0.01)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and out.abs().sum() > 0
