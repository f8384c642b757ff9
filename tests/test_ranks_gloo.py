"""Host logic of the TP linears split over GPUs, run as two real processes with
gloo on CPU.  Covered: the rank orchestration of path.py -- the row-parallel
scatter -> barrier -> reduce -> barrier sequence with its token-slice helpers,
in its reduce-scatter form and in its all-reduce form (the full output on
every rank); the whole sequence-parallel MLP block of TPRankMLP over two
layers; the LM head's gather of per-rank candidates -- with its stream barrier
and its gather.  The per-rank GPU kernels are replaced by CPU stand-ins that
do what include/tpl.h says they do; the kernels themselves are tested on the GPU in
test_gpu_ranks.py.  The results are checked against the fp64 oracle."""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O

WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _problem(batch=2, seq=8, inter=24, N=6, V=23, B=3, K=5):
    rng = np.random.default_rng(7)
    return dict(batch=batch, seq=seq, inter=inter, N=N,
                X=rng.standard_normal((batch * seq, N)),
                W1=rng.standard_normal((inter, N)) * 0.3,
                scale=rng.standard_normal(N) * 0.1,
                H=rng.standard_normal((batch * seq, inter)),
                W2=rng.standard_normal((N, inter)) * 0.1,
                bias=rng.standard_normal(N) * 0.1,
                res=rng.standard_normal((batch * seq, N)),
                x=rng.standard_normal((B, K)),
                W=np.concatenate([rng.standard_normal((V - 2, K)) * 0.1,
                                  np.zeros((2, K))]))


def _row_parallel(rank, P):
    from tensor_transformer_linear_b200 import path
    tp, batch, seq, N = WORLD, P["batch"], P["seq"], P["N"]
    part = O.partition_subparams([P["inter"]], tp, 1)
    off = sum(part.shard_width[:rank])
    k = part.shard_width[rank]
    h = torch.from_numpy(P["H"][:, off:off + k].copy())
    w = torch.from_numpy(P["W2"][:, off:off + k].copy())
    recv = torch.full((path.recv_buffer_numel(tp, batch, seq, N),), float("nan"),
                      dtype=torch.float64)
    calls = []

    def scatter(h_, w_, b_, s_, r_, tp_, addrs, stream=None):
        # what tpl_row_linear_scatter leaves in every owner's receive buffer:
        # slot r_ of rank q holds rank r_'s partial of rank q's tokens
        calls.append("scatter")
        full = h_ @ w_.T
        parts = [torch.empty_like(full) for _ in range(tp_)]
        dist.all_gather(parts, full)
        slots = recv.view(tp_, -1, N)
        for s in range(tp_):
            slots[s] = path.sp_slice(parts[s], b_, s_, tp_, rank).reshape(-1, N)

    def reduce(recv_, tp_, N_, bias_, res_, y_, stream=None):
        calls.append("reduce")
        out = recv_.view(tp_, -1, N_).sum(0)
        if bias_ is not None:
            out = out + bias_
        if res_ is not None:
            out = out + res_.reshape(-1, N_)
        return out

    barrier = path.stream_barrier()

    def counted_barrier(stream=None):
        calls.append("barrier")
        barrier(stream)

    peers = path.PeerBuffers(recv, [0] * tp)
    layer = path.TPRowParallelRank(w, rank, tp, peers, counted_barrier, scatter=scatter,
                                   reduce=reduce)
    res_slice = path.sp_slice(torch.from_numpy(P["res"]), batch, seq, tp, rank)
    y = layer(h, batch, seq, bias=torch.from_numpy(P["bias"]), residual=res_slice)
    assert calls == ["scatter", "barrier", "reduce", "barrier"]
    assert y.shape == (path.sp_rows(batch, seq, tp), N)
    return y.numpy()


def _row_allreduce(rank, P):
    from tensor_transformer_linear_b200 import path
    tp, batch, seq, N = WORLD, P["batch"], P["seq"], P["N"]
    part = O.partition_subparams([P["inter"]], tp, 1)
    off = sum(part.shard_width[:rank])
    k = part.shard_width[rank]
    h = torch.from_numpy(P["H"][:, off:off + k].copy())
    w = torch.from_numpy(P["W2"][:, off:off + k].copy())
    recv = torch.full((path.recv_buffer_numel(tp, batch, seq, N),), float("nan"),
                      dtype=torch.float64)
    out = torch.from_numpy(P["res"].copy())          # in place on the residual stream
    calls = []

    def scatter(h_, w_, b_, s_, r_, tp_, addrs, stream=None):
        calls.append("scatter")
        full = h_ @ w_.T
        parts = [torch.empty_like(full) for _ in range(tp_)]
        dist.all_gather(parts, full)
        slots = recv.view(tp_, -1, N)
        for src in range(tp_):
            slots[src] = path.sp_slice(parts[src], b_, s_, tp_, rank).reshape(-1, N)

    def reduce(recv_, tp_, b_, s_, N_, r_, addrs, bias=None, residual=None, stream=None):
        # what tpl_reduce_slots_allgather leaves in every rank's output: rank r_'s
        # token rows hold the sum of its slots + bias + its residual rows
        calls.append("reduce")
        rows = path.sp_slice(residual, b_, s_, tp_, r_).reshape(-1, N_)
        mine = recv_.view(tp_, -1, N_).sum(0) + rows
        if bias is not None:
            mine = mine + bias
        slices = [torch.empty_like(mine) for _ in range(tp_)]
        dist.all_gather(slices, mine)
        seg = s_ // tp_
        full = out.view(b_, s_, N_)
        for src in range(tp_):
            full[:, src * seg:(src + 1) * seg] = slices[src].view(b_, seg, N_)

    barrier = path.stream_barrier()

    def counted_barrier(stream=None):
        calls.append("barrier")
        barrier(stream)

    layer = path.TPRowParallelAllReduceRank(w, rank, tp, path.PeerBuffers(recv, [0] * tp),
                                            path.PeerBuffers(out, [0] * tp), counted_barrier,
                                            scatter=scatter, reduce=reduce)
    y = layer(h, batch, seq, bias=torch.from_numpy(P["bias"]), residual=out)
    assert calls == ["scatter", "barrier", "reduce", "barrier"]
    assert y.shape == (batch * seq, N)
    return y.numpy().copy()


def _mlp_block(rank, P):
    from tensor_transformer_linear_b200 import path
    tp, batch, seq, N, I = WORLD, P["batch"], P["seq"], P["N"], P["inter"]
    kr = I // tp
    w1 = torch.from_numpy(P["W1"][rank * kr:(rank + 1) * kr].copy())
    w2 = torch.from_numpy(P["W2"][:, rank * kr:(rank + 1) * kr].copy())
    rows = path.sp_rows(batch, seq, tp)
    xn = torch.full((rows, N), float("nan"), dtype=torch.float64)
    recv = torch.full((path.recv_buffer_numel(tp, batch, seq, N),), float("nan"),
                      dtype=torch.float64)

    def rmsnorm(x_, scale_, centered_, eps_, y=None, stream=None):
        y.copy_(torch.from_numpy(O.rmsnorm(x_.numpy(), scale_.numpy(), centered_, eps_)))
        return y

    def column(part_, addrs, b_, s_, w_, bias_, act_, y=None, stream=None):
        # what tpl_column_linear_gather computes from every rank's normalised slice
        parts = [torch.empty_like(xn) for _ in range(tp)]
        dist.all_gather(parts, xn)
        x_full = O.seq_gather(torch.stack(parts).numpy(), b_, s_, tp)
        return torch.from_numpy(O.activation(x_full @ w_.numpy().T, act_))

    def scatter(h_, w_, b_, s_, r_, tp_, addrs, stream=None):
        full = h_ @ w_.T
        parts = [torch.empty_like(full) for _ in range(tp_)]
        dist.all_gather(parts, full)
        slots = recv.view(tp_, -1, N)
        for src in range(tp_):
            slots[src] = path.sp_slice(parts[src], b_, s_, tp_, rank).reshape(-1, N)

    def reduce(recv_, tp_, N_, bias_, res_, y_, stream=None):
        y_.copy_(recv_.view(tp_, -1, N_).sum(0) + res_)
        return y_

    block = path.TPRankMLP(w1, w2, rank, tp, "gelu_erf", path.PeerBuffers(xn, [0] * tp),
                           path.PeerBuffers(recv, [0] * tp), path.stream_barrier(),
                           scale=torch.from_numpy(P["scale"]), centered=True,
                           ops=dict(rmsnorm=rmsnorm, column=column, scatter=scatter,
                                    reduce=reduce))
    x = path.sp_slice(torch.from_numpy(P["X"]), batch, seq, tp, rank).reshape(rows, N)
    for _ in range(2):                       # two layers sharing the weights
        block(x, batch, seq)
    return x.numpy()


def _lmhead(rank, P):
    from tensor_transformer_linear_b200 import path
    tp, V = WORLD, P["W"].shape[0]
    shard = -(-V // tp)
    lo, hi = rank * shard, min(V, (rank + 1) * shard)
    x, wl = P["x"], P["W"][lo:hi]

    def local_argmax(x_, stream=None):
        # what tpl_lmhead_argmax over this slice returns: (max, slice-local id)
        lg = np.asarray(x_) @ wl.T
        return (torch.from_numpy(lg.max(axis=1)),
                torch.from_numpy(lg.argmax(axis=1).astype(np.int32)))

    def merge(m, i, stride, stream=None):
        # what tpl_argmax_merge computes: larger logit, then lower global id
        m, i = m.numpy(), i.numpy()
        ids = []
        for b in range(m.shape[1]):
            cands = [(-m[s, b], s * stride + int(i[s, b])) for s in range(m.shape[0])
                     if i[s, b] >= 0]
            ids.append(min(cands)[1])
        return np.array(ids)

    head = path.TPLMHeadRank(torch.from_numpy(wl), rank, tp, shard, local_argmax=local_argmax,
                             merge=merge)
    return head(x)


def _worker(rank, port, P, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out[(rank, "row")] = _row_parallel(rank, P)
        out[(rank, "allreduce")] = _row_allreduce(rank, P)
        out[(rank, "mlp")] = _mlp_block(rank, P)
        out[(rank, "lm")] = _lmhead(rank, P)
    finally:
        dist.destroy_process_group()


def test_rank_orchestration_over_two_processes():
    P = _problem()
    # an exact tie across the two ranks' vocab slices for batch row 1
    shard = -(-P["W"].shape[0] // WORLD)
    P["W"][shard + 3] = P["W"][4] = 5.0 * P["x"][1] / np.linalg.norm(P["x"][1])
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, P, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0

    batch, seq, tp = P["batch"], P["seq"], WORLD
    part = O.partition_subparams([P["inter"]], tp, 1)
    h_parts, off = [], 0
    for k in part.shard_width:
        h_parts.append(P["H"][:, off:off + k])
        off += k
    ref = O.row_linear_reduce_scatter(h_parts, O.row_weight_slices(P["W2"], part.shard_width),
                                      batch, seq, bias=P["bias"],
                                      residual_sp=O.seq_scatter(P["res"], batch, seq, tp))
    for r in range(tp):
        got = out[(r, "row")].reshape(batch, seq // tp, -1)
        assert np.allclose(got, ref[r], rtol=1e-12, atol=1e-12)

    ref_full = O.row_linear_reduce(h_parts, O.row_weight_slices(P["W2"], part.shard_width),
                                   P["bias"], P["res"])
    for r in range(tp):
        assert np.allclose(out[(r, "allreduce")], ref_full, rtol=1e-12, atol=1e-12)

    x = P["X"]
    for _ in range(2):
        x = O.tp_mlp(x, P["W1"], P["W2"], tp, "gelu_erf", scale=P["scale"], centered=True,
                     norm=True, residual=True)
    ref_mlp = O.seq_scatter(x, batch, seq, tp)
    for r in range(tp):
        got = out[(r, "mlp")].reshape(batch, seq // tp, -1)
        assert np.allclose(got, ref_mlp[r], rtol=1e-12, atol=1e-12)

    lm = O.lmhead_argmax(P["x"], P["W"], tp, 1)
    for r in range(tp):
        assert list(out[(r, "lm")]) == [int(v) for v in lm.ids]
    assert int(lm.ids[1]) == 4          # the tie went to the lower global id


def _leaver_worker(rank, port, step1_done, out):
    """Both ranks run one row-parallel step; then rank 1 leaves (between steps,
    nothing in flight) and rank 0 runs the next step, whose barrier must end with
    an error within the process-group timeout instead of waiting for good."""
    import time
    from tensor_transformer_linear_b200 import path
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=5))
    batch, seq, N, k = 1, 4, 3, 2
    recv = torch.zeros(path.recv_buffer_numel(WORLD, batch, seq, N), dtype=torch.float64)

    def scatter(h_, w_, b_, s_, r_, tp_, addrs, stream=None):
        pass                                    # the exchange itself is not under test

    def reduce(recv_, tp_, N_, bias_, res_, y_, stream=None):
        return recv_.view(tp_, -1, N_).sum(0)

    layer = path.TPRowParallelRank(torch.ones(N, k, dtype=torch.float64), rank, WORLD,
                                   path.PeerBuffers(recv, [0] * WORLD), path.stream_barrier(),
                                   scatter=scatter, reduce=reduce)
    h = torch.ones(batch * seq, k, dtype=torch.float64)
    layer(h, batch, seq)
    if rank == 1:
        step1_done.wait(30)
        os._exit(0)                             # leaves without a word to rank 0
    step1_done.set()
    time.sleep(0.5)
    t0 = time.monotonic()
    try:
        layer(h, batch, seq)
        out["result"] = "returned"
    except Exception as e:                      # gloo reports the lost peer or the timeout
        out["result"] = "error"
        out["kind"] = type(e).__name__
    out["seconds"] = time.monotonic() - t0
    os._exit(0)                                 # the group cannot be torn down cleanly


def test_a_rank_that_leaves_ends_the_next_barrier_with_an_error():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    step1_done = ctx.Event()
    port = _free_port()
    procs = [ctx.Process(target=_leaver_worker, args=(r, port, step1_done, out))
             for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out.get("result") == "error", dict(out)
    assert out["seconds"] < 30, dict(out)
