"""The LM-head entry point that allocates nothing (tpl_lmhead_argmax_static).

Some callers cannot allocate device memory -- a plugin inside a host
framework that owns all device memory and passes in only its input and output
buffers, or a latency-critical decode loop where an allocation, which can
synchronise the device, is not allowed.  tpl_lmhead_argmax_static serves them:
its scratch is a fixed array inside the library.  This test calls it through
the C ABI twice in a row (the second call reuses the scratch the first one
left behind) and checks each result against tpl_lmhead_argmax with a
caller-provided workspace.  It sits in a file of its own that pytest collects
last.
"""
import numpy as np
import pytest
import torch

import tensor_transformer_linear_b200 as T
from workloads import gen

from ._parity import TOL_BF16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,K,V,tp,nc", [(32, 4096, 20000, 8, 4), (5, 256, 1000, 3, 2)])
def test_static_scratch_matches_workspace_entry_point(B, K, V, tp, nc):
    dev = "cuda"
    x = gen.normal((B, K), 1.0, tensor_id=0, seed=7, device=dev)
    w = gen.normal((V, K), 0.02, tensor_id=1, seed=7, device=dev)
    ws = T.lmhead_workspace(B, V, tp, nc, dev)
    ref_logits = torch.empty(B * V, dtype=torch.float32, device=dev)
    ids_r, max_r, idx_r = T.tpl_lmhead_argmax(x, w, tp, nc, ws, logits=ref_logits)
    for call in range(2):
        logits = torch.full((B * V,), float("nan"), dtype=torch.float32, device=dev)
        ids, smax, sidx = T.tpl_lmhead_argmax_static(x, w, tp, nc, logits=logits)
        torch.cuda.synchronize()
        assert T.tpl_get_device_status() == 0
        assert torch.equal(ids, ids_r), call
        assert torch.equal(sidx, idx_r), call
        g, r = smax.double().cpu().numpy(), max_r.double().cpu().numpy()
        assert np.linalg.norm(g - r) <= TOL_BF16 * np.linalg.norm(r), call
        g, r = logits.double().cpu().numpy(), ref_logits.double().cpu().numpy()
        assert np.linalg.norm(g - r) <= TOL_BF16 * np.linalg.norm(r), call


def test_static_scratch_rejects_sizes_beyond_its_limit():
    dev = "cuda"
    x = torch.zeros((256, 64), dtype=torch.bfloat16, device=dev)
    w = torch.zeros((64 * 64, 64), dtype=torch.bfloat16, device=dev)
    with pytest.raises(T.TplError) as e:          # 64 shards x 256 rows of keys > 64 KiB
        T.tpl_lmhead_argmax_static(x, w, 64, 1)
    assert e.value.name == "TPL_ERR_SHAPE"
