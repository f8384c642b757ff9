"""The TP linears split over GPUs, run by two real processes on one GPU.

Each process is one rank (gloo process group on the host).  The ranks' peer
buffers -- the RMSNorm output slices the gathered c_fc reads, the receive
buffers the scattered c_proj writes into, the full outputs of the all-reduce
form -- are exported as CUDA IPC handles and opened by the other process
(path.exchange_peer_buffers), exactly as on several GPUs; here both mappings
point into the same device.  Every step runs the library's kernels; the ranks
are ordered only by host-side barriers (the stream is synchronised, then the
group's barrier), so no kernel ever waits on another process.

Covered, against the fp64 oracle (relative Frobenius and element-wise bounds):
  * two layers of the sequence-parallel MLP block (TPRankMLP: RMSNorm of the
    rank's token slice -> c_fc + GELU over every rank's slice, read through the
    peer mappings -> c_proj partials scattered into the owners' receive
    buffers -> slots summed with the residual, in place);
  * the all-reduce form of the row-parallel linear (TPRowParallelAllReduceRank:
    every rank ends with the full output, written by the peers' stores);
  * the LM head split over the ranks (TPLMHeadRank), candidates gathered on
    the host and merged on the device.
"""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch

import oracle as O
from workloads import gen

from . import _bounds as Bd
from ._parity import TOL_BF16, check_ids, f64, rel

pytestmark = pytest.mark.gpu

TP, BATCH, SEQ, H, I = 2, 2, 256, 256, 1024     # token slices of 128 rows per sequence
N2, K2 = 384, 512                                # the all-reduce row linear
LM_B, LM_K, LM_V = 8, 256, 5000
LAYERS = 2


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _inputs():
    """Host tensors (bf16), the same in every process and in the oracle."""
    M = BATCH * SEQ
    t = {"x": gen.normal((M, H), 1.0, tensor_id=0, seed=11),
         "scale": gen.normal((H,), 0.1, tensor_id=4, seed=11, dtype=torch.float32),
         "h2": gen.normal((M, K2), 1.0, tensor_id=5, seed=11),
         "w2b": gen.normal((N2, K2), 0.05, tensor_id=6, seed=11),
         "bias2": gen.normal((N2,), 0.05, tensor_id=7, seed=11),
         "res2": gen.normal((M, N2), 1.0, tensor_id=8, seed=11),
         "lx": gen.normal((LM_B, LM_K), 1.0, tensor_id=9, seed=11),
         "lw": gen.normal((LM_V, LM_K), 0.05, tensor_id=10, seed=11)}
    for l in range(LAYERS):
        t[f"w1_{l}"] = gen.normal((I, H), 0.05, tensor_id=1 + 16 * l, seed=11)
        t[f"w2_{l}"] = gen.normal((H, I), 0.05, tensor_id=2 + 16 * l, seed=11)
    return t


def _rank(rank, port, out_dir):
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=TP, timeout=datetime.timedelta(seconds=120))
    try:
        import tensor_transformer_linear_b200 as T
        from tensor_transformer_linear_b200 import path
        t = _inputs()
        M, kr = BATCH * SEQ, I // TP
        stream = torch.cuda.current_stream()

        def barrier(s=None):
            (s or stream).synchronize()
            dist.barrier()

        # --- sequence-parallel MLP block, two layers, in place on the token slice
        x_slice = path.sp_slice(t["x"], BATCH, SEQ, TP, rank).reshape(-1, H).to(dev)
        xn = path.exchange_peer_buffers(torch.empty_like(x_slice))
        recv = path.exchange_peer_buffers(
            torch.empty(path.recv_buffer_numel(TP, BATCH, SEQ, H), dtype=torch.bfloat16,
                        device=dev))
        scale = t["scale"].to(dev)
        for l in range(LAYERS):
            w1s = t[f"w1_{l}"][rank * kr:(rank + 1) * kr].contiguous().to(dev)
            w2s = t[f"w2_{l}"][:, rank * kr:(rank + 1) * kr].contiguous().to(dev)
            blk = path.TPRankMLP(w1s, w2s, rank, TP, "gelu_erf", xn, recv, barrier,
                                 scale=scale, centered=True)
            blk(x_slice, BATCH, SEQ)
        barrier()
        mlp_out = x_slice.cpu()

        # --- row-parallel linear with the full output on every rank
        k2 = K2 // TP
        h_r = t["h2"][:, rank * k2:(rank + 1) * k2].contiguous().to(dev)
        w_r = t["w2b"][:, rank * k2:(rank + 1) * k2].contiguous().to(dev)
        recv2 = path.exchange_peer_buffers(
            torch.empty(path.recv_buffer_numel(TP, BATCH, SEQ, N2), dtype=torch.bfloat16,
                        device=dev))
        out2 = path.exchange_peer_buffers(t["res2"].to(dev))   # in place on the residual
        row = path.TPRowParallelAllReduceRank(w_r, rank, TP, recv2, out2, barrier)
        row(h_r, BATCH, SEQ, bias=t["bias2"].to(dev), residual=out2.local)
        barrier()
        row_out = out2.local.cpu()

        # --- LM head over the ranks' vocab slices; candidates gathered on the host
        shard = -(-LM_V // TP)
        w_slice = t["lw"][rank * shard:min(LM_V, (rank + 1) * shard)].contiguous().to(dev)

        def host_gather(v, stream=None):
            parts = [torch.empty_like(v.cpu()) for _ in range(TP)]
            (stream or torch.cuda.current_stream()).synchronize()
            dist.all_gather(parts, v.cpu())
            return torch.stack(parts).to(dev)

        lm = path.TPLMHeadRank(w_slice, rank, TP, shard, gather=host_gather)
        ids = lm(t["lx"].to(dev)).cpu()
        assert T.tpl_get_device_status() == 0
        torch.save({"mlp": mlp_out, "row": row_out, "ids": ids},
                   os.path.join(out_dir, f"rank{rank}.pt"))
        barrier()
    finally:
        dist.destroy_process_group()


def test_two_processes_one_gpu_peer_buffers_over_ipc():
    import torch.multiprocessing as mp
    with tempfile.TemporaryDirectory() as d:
        ctx = mp.get_context("spawn")
        port = _port()
        procs = [ctx.Process(target=_rank, args=(r, port, d)) for r in range(TP)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        codes = [p.exitcode for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        assert codes == [0, 0], codes
        got = [torch.load(os.path.join(d, f"rank{r}.pt")) for r in range(TP)]

    t = _inputs()
    M = BATCH * SEQ
    # the block, two layers, every token; each rank holds its token slices
    xr = f64(t["x"])
    proxy = None
    for l in range(LAYERS):
        y, own, car = Bd.rank_mlp(xr, f64(t[f"w1_{l}"]), f64(t[f"w2_{l}"]), TP, "gelu_erf",
                                  scale=f64(t["scale"]), centered=True, x_proxy=proxy)
        if l + 1 < LAYERS:
            proxy = Bd.stored(y, own, car, Bd.U_BF16)
        xr = y
    ref_sp = O.seq_scatter(xr, BATCH, SEQ, TP)
    own_sp, car_sp = O.seq_scatter(own, BATCH, SEQ, TP), O.seq_scatter(car, BATCH, SEQ, TP)
    for r in range(TP):
        g = f64(got[r]["mlp"]).reshape(BATCH, SEQ // TP, H)
        assert rel(g, ref_sp[r]) <= TOL_BF16, r
        Bd.check(g, ref_sp[r], own_sp[r], car_sp[r], what=f"mlp rank {r}")

    # the all-reduce form: the full output on every rank, the same bits on both
    k2 = K2 // TP
    hs = [f64(t["h2"])[:, r * k2:(r + 1) * k2] for r in range(TP)]
    ws = [f64(t["w2b"])[:, r * k2:(r + 1) * k2] for r in range(TP)]
    ref, own, car = Bd.scatter_reduce(hs, ws, f64(t["bias2"]), f64(t["res2"]))
    for r in range(TP):
        assert rel(got[r]["row"], ref) <= TOL_BF16, r
        Bd.check(f64(got[r]["row"]), ref, own, car, what=f"row rank {r}")
    assert torch.equal(got[0]["row"], got[1]["row"])

    # the LM head: merged global ids, the same on both ranks
    res = O.lmhead_argmax(f64(t["lx"]), f64(t["lw"]), TP, 1)
    for r in range(TP):
        check_ids(got[r]["ids"].numpy(), res)
    assert torch.equal(got[0]["ids"], got[1]["ids"])
    assert M == BATCH * SEQ
