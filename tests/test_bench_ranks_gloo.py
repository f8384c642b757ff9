"""bench.py's TP-rank mode (``--workload tp_ranks`` under torchrun, one rank
per GPU) as two gloo processes on CPU.

Each process builds ``bench.RankTP`` for its rank, with CPU stand-ins for the
library calls, the peer mapping and the stream barrier (what include/tpl.h
says the calls do, as in test_ranks_gloo.py), and runs two steps of the MLP
block in place on its token slice.  Checked: the slices against the fp64
oracle, the work accounting (the job's FLOPs per step, this rank's GEMM
FLOPs) and the line's config for both arms.
"""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from workloads import configs as C

WORLD = 2
SMALL = C.MLPWorkload("small", batch=2, seq=8, hidden=6, inter=24, tp=WORLD, act="gelu_erf",
                      w_sigma=0.3, dtype=torch.float64, norm=True, norm_scale=True,
                      residual=True)


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from tensor_transformer_linear_b200 import path
        m, tp = SMALL, WORLD
        bufs = []

        def exchange(t):
            bufs.append(t)      # bufs[0]: the normalised slice, bufs[1]: the receive buffer
            return path.PeerBuffers(t, [0] * tp)

        def rmsnorm(x_, scale_, centered_, eps_, y=None, stream=None):
            y.copy_(torch.from_numpy(O.rmsnorm(x_.numpy(), scale_.double().numpy(), centered_,
                                               eps_)))
            return y

        def column(part_, addrs, b_, s_, w_, bias_, act_, y=None, stream=None):
            xn = bufs[0]
            parts = [torch.empty_like(xn) for _ in range(tp)]
            dist.all_gather(parts, xn)
            x_full = O.seq_gather(torch.stack(parts).numpy(), b_, s_, tp)
            return torch.from_numpy(O.activation(x_full @ w_.numpy().T, act_))

        def scatter(h_, w_, b_, s_, r_, tp_, addrs, stream=None):
            full = h_ @ w_.T
            parts = [torch.empty_like(full) for _ in range(tp_)]
            dist.all_gather(parts, full)
            slots = bufs[1].view(tp_, -1, m.hidden)
            for src in range(tp_):
                slots[src] = path.sp_slice(parts[src], b_, s_, tp_, rank).reshape(-1, m.hidden)

        def reduce(recv_, tp_, N_, bias_, res_, y_, stream=None):
            y_.copy_(recv_.view(tp_, -1, N_).sum(0) + res_)
            return y_

        def reduce_norm(recv_, tp_, N_, xn_, scale_, centered_, eps_, bias_, res_, y_,
                        stream=None):
            reduce(recv_, tp_, N_, bias_, res_, y_)
            xn_.copy_(torch.from_numpy(O.rmsnorm(y_.numpy(), scale_.double().numpy(),
                                                 centered_, eps_)))
            return y_

        wl = bench.RankTP("cpu", rank, WORLD, workload=m, exchange=exchange,
                          barrier=path.stream_barrier(),
                          ops=dict(rmsnorm=rmsnorm, column=column, scatter=scatter,
                                   reduce=reduce, reduce_norm=reduce_norm))
        calls = []
        wl.block.rmsnorm = lambda *a, **k: (calls.append("rmsnorm"), rmsnorm(*a, **k))[1]
        for _ in range(2):
            wl.step(None)
        # the second step's RMSNorm came out of the first step's slot reduction
        assert calls == ["rmsnorm"]
        wl.inputs_replaced()
        wl.step(None)
        assert calls == ["rmsnorm", "rmsnorm"]
        out[rank] = (wl.x.numpy().copy(), wl.flops, wl.gemm_flops, wl.parts,
                     wl.gemm_part_ids())
    finally:
        dist.destroy_process_group()


def test_rank_mode_of_the_bench_over_two_processes():
    import bench
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert [p.exitcode for p in procs] == [0, 0]

    m = SMALL
    x = C.mlp_x(m).numpy()
    w1, w2, s = C.mlp_w1(m).numpy(), C.mlp_w2(m).numpy(), C.mlp_scale(m).double().numpy()
    ref = x
    for _ in range(3):            # three steps with the same weights, in place
        ref = O.tp_mlp(ref, w1, w2, WORLD, m.act, scale=s, centered=True, norm=True,
                       residual=True)
    ref_sp = O.seq_scatter(ref, m.batch, m.seq, WORLD)
    for r in range(WORLD):
        got, flops, gflops, parts, gids = out[r]
        np.testing.assert_allclose(got.reshape(ref_sp[r].shape), ref_sp[r], rtol=1e-12,
                                   atol=1e-12)
        assert flops == 4.0 * m.M * m.hidden * m.inter       # the whole job, once per step
        assert gflops == flops / WORLD
        assert [parts[i] for i in gids] == ["rank_column_gather", "rank_row_scatter"]
    # both arms print the same config for the rank mode
    cfg = bench.workload_config("tp_ranks", WORLD)
    assert "one TP rank per GPU" in cfg["parallelism"] and "2 ranks" in cfg["workload"]
    assert bench.workload_config("tp_ranks", 1)["workload"] == bench.WORKLOAD_NAMES["tp_ranks"]
