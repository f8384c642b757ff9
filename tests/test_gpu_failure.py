"""Failure detection on the GPU without a fault: a bounded pipeline wait that
runs out reports TPL_ERR_TIMEOUT through the status word, and the context stays
usable for the next (correct) call."""
import pytest
import torch

import oracle as O
import tensor_transformer_linear_b200 as T
from workloads import gen

from ._parity import TOL_BF16, f64, rel

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert T.tpl_get_device_status() == 0
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    T.tpl_selftest_wait_timeout(20_000_000, waited)          # 20 ms, nothing ever arrives
    assert T.tpl_get_device_status() == 7                      # TPL_ERR_TIMEOUT, then cleared
    assert T.tpl_get_device_status() == 0
    assert 20_000 <= int(waited.item()) < 1_000_000
    # the next call runs normally
    x = gen.normal((200, 128), 1.0, tensor_id=0)
    w = gen.normal((256, 128), 0.05, tensor_id=1)
    p = T.tpl_partition_subparams([256], 2, 1)
    y = T.tpl_column_linear(p, x.cuda(), w.cuda(), None, "gelu_erf")
    torch.cuda.synchronize()
    ref = O.column_linear(f64(x), f64(w), None, O.partition_subparams([256], 2, 1), "gelu_erf")
    for g, r in zip(T.shard_views(y, p, 200), ref):
        assert rel(g, r) <= TOL_BF16
    assert T.tpl_get_device_status() == 0
