"""Per-CTA timing records of the tensor-core kernels (tpl_trace_set).

With a trace buffer installed, each CTA of the single-CTA GEMM, the CTA-pair
GEMM and the LM head leaves one record: the launch number (tpl_launch_count
before the launch), its kind, its CTA index, globaltimer at start and end and
the SM cycles between.  Checked: one record per CTA of every launch, the
launch numbers, ordered and plausible times and clocks, nothing recorded with
the buffer removed, and overflow dropping records but counting them.  The
kernels' results are unchanged by tracing."""
import pytest
import torch

import tensor_transformer_linear_b200 as T
from workloads import gen

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _t(shape, sigma, tid):
    return gen.normal(shape, sigma, tensor_id=tid, seed=5, dtype=torch.bfloat16).to(DEV)


def _launches():
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    p = T.tpl_partition_subparams([1024], 4, 1)
    small, big = _t((96, 512), 1.0, 0), _t((1024, 512), 1.0, 1)
    w = _t((1024, 512), 0.02, 2)
    xl, wl = _t((8, 1024), 1.0, 3), _t((4000, 1024), 0.02, 4)
    ws = T.lmhead_workspace(8, 4000, 2, 2, DEV)
    runs = [
        ("gemm", lambda: T.tpl_column_linear(p, small, w, None, "none")),
        ("gemm_pair", lambda: T.tpl_column_linear(p, big, w, None, "gelu_erf")),
        ("lmhead", lambda: T.tpl_lmhead_argmax(xl, wl, 2, 2, ws)),
    ]
    return runs, sm


def test_trace_records_every_cta_of_every_launch():
    runs, sm = _launches()
    ref = [fn() for _, fn in runs]
    torch.cuda.synchronize()
    seqs = []
    with T.Trace(4096, DEV) as tr:
        got = []
        for _, fn in runs:
            seqs.append(T.tpl_launch_count())
            got.append(fn())
        torch.cuda.synchronize()
    assert T.tpl_get_device_status() == 0
    # tracing leaves the results alone
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    assert torch.equal(got[2][0], ref[2][0])
    L = tr.launches()
    assert [l["seq"] for l in L] == seqs
    assert [l["kind"] for l in L] == [k for k, _ in runs]
    recs = tr.records()
    for l in L:
        ctas = sorted(r[2] for r in recs if r[0] == l["seq"])
        assert ctas == list(range(len(ctas))) and 1 <= len(ctas) <= sm
        assert 0 < l["cta_us"] <= l["span_us"] < 1e5
        assert 300.0 < l["sm_mhz"] < 2500.0
    assert all(r[4] > r[3] and r[5] > 0 for r in recs)
    assert tr.dropped() == 0
    # removed: nothing more is recorded
    n = len(recs)
    runs[1][1]()
    torch.cuda.synchronize()
    assert len(tr.records()) == n


def test_trace_overflow_counts_dropped_records():
    runs, _ = _launches()
    with T.Trace(3, DEV) as tr:
        runs[1][1]()
        torch.cuda.synchronize()
    assert len(tr.records()) == 3
    assert tr.dropped() > 0
