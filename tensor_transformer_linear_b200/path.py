"""The sharded-linear path composed from the C-ABI calls.

Layout helpers (views and one-time weight packing, done with torch as plain
data movement) and the block orchestration: RMSNorm -> column-parallel c_fc
with GELU -> row-parallel c_proj with the partial-sum reduction (and the
residual) fused in, per the nanotron "MLP Module" and the google-research
residual section.  Each step is one call into libtpl.so.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch

from ._tpl import (Partition, TplError, tpl_argmax_merge, tpl_column_linear,
                   tpl_column_linear_gather, tpl_column_linear_rmsnorm,
                   tpl_column_linear_rmsnorm_workspace_size, tpl_fold_norm_scale,
                   tpl_get_device_status, tpl_lmhead_argmax,
                   tpl_lmhead_workspace_size, tpl_partition_subparams, tpl_reduce_slots,
                   tpl_reduce_slots_allgather, tpl_reduce_slots_rmsnorm, tpl_rmsnorm,
                   tpl_row_linear_reduce,
                   tpl_row_linear_scatter, tpl_tp_mlp_fp32)


def shard_views(y: torch.Tensor, p: Partition, M: int) -> List[torch.Tensor]:
    """Rank r's ``[M, shard_width[r]]`` view of a column-linear output buffer."""
    out = []
    for r in range(p.tp_size):
        base, w = M * p.shard_base[r], p.shard_width[r]
        out.append(y.view(-1)[base:base + M * w].view(M, w))
    return out


def pack_row_weight(w2_full: torch.Tensor, k_w: Sequence[int]) -> torch.Tensor:
    """Rank-major packing of an unsharded ``[N, K]`` c_proj weight.

    Rank r's block ``[N, k_w[r]]`` holds columns ``sum(k_w[:r]) ..`` of the
    weight, i.e. the slice that rank holds in a row-parallel layout.
    """
    blocks, off = [], 0
    for k in k_w:
        blocks.append(w2_full[:, off:off + k].contiguous().view(-1))
        off += k
    return torch.cat(blocks)


class TPMLP:
    """One TP MLP block: ``[x +] c_proj(act(c_fc(rmsnorm(x))))``, all shards on one GPU.

    ``fused_norm``: the RMSNorm runs inside the c_fc GEMM
    (tpl_column_linear_rmsnorm): its scale is folded into W1 here, once, and no
    normalised copy of x is written.  Otherwise tpl_rmsnorm writes one first.
    """

    def __init__(self, w1: torch.Tensor, w2_full: torch.Tensor, tp: int, act: str,
                 scale: Optional[torch.Tensor] = None, centered: bool = False,
                 norm: bool = True, residual: bool = False, eps: float = 1e-6,
                 fused_norm: bool = False, fused_fp32: bool = True):
        self.inter, self.hidden = w1.shape
        self.part = tpl_partition_subparams([self.inter], tp, 1)
        self.k_w = [self.part.shard_width[r] for r in range(tp)]
        self.w1 = w1.contiguous()
        self.w2 = pack_row_weight(w2_full, self.k_w)
        self.act, self.scale, self.centered = act, scale, centered
        self.norm, self.residual, self.eps = norm, residual, eps
        self.fused_norm = bool(fused_norm and norm)
        if self.fused_norm and scale is not None:
            self.w1 = tpl_fold_norm_scale(self.w1, scale, centered)
        self._bufs = {}
        self._norm_ws = None
        # fp32 blocks without a norm: the whole block in one launch
        # (tpl_tp_mlp_fp32) when the kernel takes the shapes
        self.fused_fp32 = bool(fused_fp32 and not norm and w1.dtype == torch.float32)

    def _buf(self, name, numel, like):
        b = self._bufs.get(name)
        if b is None or b.numel() < numel or b.dtype != like.dtype or b.device != like.device:
            b = torch.empty(numel, dtype=like.dtype, device=like.device)
            self._bufs[name] = b
        return b[:numel]

    def norm_workspace(self, M: int, device) -> torch.Tensor:
        """The fused norm's workspace for M rows (zero-filled when it grows)."""
        need = tpl_column_linear_rmsnorm_workspace_size(M)
        if self._norm_ws is None or self._norm_ws.numel() < need:
            self._norm_ws = torch.zeros(need, dtype=torch.uint8, device=device)
        return self._norm_ws

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
        M = x.numel() // self.hidden
        if self.fused_fp32:
            if out is None:
                out = torch.empty((M, self.hidden), dtype=x.dtype, device=x.device)
            try:
                return tpl_tp_mlp_fp32(x.view(M, self.hidden), self.w1, self.w2,
                                       self.part.tp_size, self.act,
                                       residual=x.view(M, self.hidden) if self.residual else None,
                                       y=out, stream=stream)
            except TplError as e:
                if e.name not in ("TPL_ERR_UNSUPPORTED", "TPL_ERR_INDIVISIBLE"):
                    raise
                self.fused_fp32 = False     # shapes outside the fused kernel: two launches
        if self.fused_norm:
            h = self._buf("h", M * self.inter, x)
            ws = self.norm_workspace(M, x.device)
            tpl_column_linear_rmsnorm(self.part, x.view(M, self.hidden), self.w1, None, self.eps,
                                      self.act, ws, y=h, stream=stream)
            if out is None:
                out = torch.empty((M, self.hidden), dtype=x.dtype, device=x.device)
            tpl_row_linear_reduce(h, self.k_w, M, self.w2, None,
                                  x.view(M, self.hidden) if self.residual else None, y=out,
                                  stream=stream)
            return out
        xn = x
        if self.norm:
            xn = self._buf("xn", x.numel(), x).view(M, self.hidden)
            tpl_rmsnorm(x.view(M, self.hidden), self.scale, self.centered, self.eps, y=xn,
                        stream=stream)
        h = self._buf("h", M * self.inter, x)
        tpl_column_linear(self.part, xn.view(M, self.hidden), self.w1, None, self.act, y=h,
                          stream=stream)
        if out is None:
            out = torch.empty((M, self.hidden), dtype=x.dtype, device=x.device)
        tpl_row_linear_reduce(h, self.k_w, M, self.w2, None,
                              x.view(M, self.hidden) if self.residual else None, y=out,
                              stream=stream)
        return out


class TPStack:
    """``x <- x + MLP(RMSNorm(x))`` over several layers, in place on x."""

    def __init__(self, layers: Sequence[TPMLP]):
        self.layers = list(layers)

    def __call__(self, x: torch.Tensor, stream=None):
        for layer in self.layers:
            layer(x, out=x, stream=stream)
        return x


# ---------------------------------------------------------------------------
# The TP linears split over GPUs: one process per GPU, rank `rank` of `tp`.
# ---------------------------------------------------------------------------

def sp_rows(batch: int, seq: int, tp: int) -> int:
    """Token rows a rank owns after the reduce-scatter: ``batch * seq / tp``
    (nanotron "MLP Module": ``[batch, seq // tp, hidden]`` per rank)."""
    if seq % tp != 0:
        raise ValueError(f"seq {seq} is not divisible by tp {tp}")
    return batch * (seq // tp)


def sp_token_owner(t: int, seq: int, tp: int) -> int:
    """The rank that owns token ``t`` of every sequence."""
    return t // (seq // tp)


def sp_slice(x: torch.Tensor, batch: int, seq: int, tp: int, rank: int) -> torch.Tensor:
    """Rank ``rank``'s token slice ``[batch, seq/tp, N]`` of a ``[batch*seq, N]``
    tensor, contiguous (e.g. its share of the residual stream)."""
    n = x.shape[-1]
    return x.reshape(batch, tp, seq // tp, n)[:, rank].contiguous()


def recv_buffer_numel(tp: int, batch: int, seq: int, N: int) -> int:
    """Elements of one rank's receive buffer ``[tp][batch][seq/tp][N]``: one slot
    per source rank, each that source's partial of this rank's tokens."""
    return tp * sp_rows(batch, seq, tp) * N


class PeerBuffers:
    """This rank's receive buffer and the device address of every rank's receive
    buffer as mapped into this process (``addrs[rank]`` is the local one)."""

    def __init__(self, local: torch.Tensor, addrs: Sequence[int], keep: Sequence = ()):
        self.local = local
        self.addrs = [int(a) for a in addrs]
        self._keep = list(keep)  # mapped peer storages stay open while in use


def local_peer_buffers(bufs: Sequence[torch.Tensor], rank: int) -> PeerBuffers:
    """Every rank's buffer lives in this process (ranks run one after another)."""
    return PeerBuffers(bufs[rank], [b.data_ptr() for b in bufs])


def exchange_peer_buffers(local: torch.Tensor, group=None) -> PeerBuffers:
    """Maps every rank's receive buffer into this process.

    One process per GPU on one node with peer access between the GPUs: each rank
    exports its buffer's storage as a CUDA IPC handle, the handles are
    all-gathered over the process group, and each peer storage is opened here.
    Plain peer mappings only: nothing is bound to a multicast object.
    """
    import torch.distributed as dist
    st = local.untyped_storage()
    handle = st._share_cuda_()
    offset = local.data_ptr() - st.data_ptr()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    got = [None] * world
    dist.all_gather_object(got, (handle, offset), group=group)
    addrs, keep = [], []
    for q, (h, off) in enumerate(got):
        if q == rank:
            addrs.append(local.data_ptr())
            continue
        peer = torch.UntypedStorage._new_shared_cuda(*h)
        keep.append(peer)
        addrs.append(peer.data_ptr() + off)
    return PeerBuffers(local, addrs, keep)


def stream_barrier(group=None, device=None) -> Callable:
    """A barrier ordered on a stream: an all-reduce of one element over the
    group, enqueued on the stream.  Work after it on that stream starts only when
    every rank's work before its own barrier has completed, which is what makes
    the peer writes of every rank's scatter visible to the readers."""
    import torch.distributed as dist
    token = torch.zeros(1, dtype=torch.int32, device=device)

    def barrier(stream=None):
        if stream is None:
            dist.all_reduce(token, group=group)
        else:
            with torch.cuda.stream(stream):
                dist.all_reduce(token, group=group)
    return barrier


class TPRowParallelRank:
    """Rank ``rank``'s row-parallel linear over ``tp`` GPUs, reduced by a
    reduce-scatter along the sequence (google-research: each shard's partial,
    reduced afterwards; nanotron "MLP Module": ``[batch, seq // tp, hidden]``).

    Each call: scatter (this rank's partial, written by the GEMM epilogue into
    every owner's receive buffer) -> barrier -> reduce this rank's slots (+ bias,
    + residual) -> barrier.  The first barrier makes every partial visible before
    any rank reads its slots; the second keeps the next call's scatter from
    overwriting slots a slower rank is still reading.

    ``w_shard`` is ``[N, k]``, this rank's columns of the unsharded weight.
    ``scatter`` and ``reduce`` default to the library's calls.
    """

    def __init__(self, w_shard: torch.Tensor, rank: int, tp: int, peers: PeerBuffers,
                 barrier: Callable, scatter: Optional[Callable] = None,
                 reduce: Optional[Callable] = None):
        self.w = w_shard.contiguous()
        self.rank, self.tp, self.peers, self.barrier = rank, tp, peers, barrier
        self.scatter = scatter or tpl_row_linear_scatter
        self.reduce = reduce or tpl_reduce_slots

    def __call__(self, h_shard: torch.Tensor, batch: int, seq: int,
                 bias: Optional[torch.Tensor] = None, residual: Optional[torch.Tensor] = None,
                 y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """``h_shard`` ``[batch*seq, k]``; ``residual`` this rank's token slice
        ``[batch*seq/tp, N]`` (see :func:`sp_slice`).  Returns that slice of Y."""
        N = self.w.shape[0]
        sp_rows(batch, seq, self.tp)
        self.scatter(h_shard, self.w, batch, seq, self.rank, self.tp, self.peers.addrs,
                     stream=stream)
        self.barrier(stream)
        out = self.reduce(self.peers.local, self.tp, N, bias, residual, y, stream=stream)
        self.barrier(stream)
        return out


class TPRowParallelAllReduceRank:
    """Rank ``rank``'s row-parallel linear over ``tp`` GPUs with the full output
    on every rank (google-research: the partials reduced over the sharded
    contraction axis; nanotron "MLP Module" without sequence parallelism).

    Each call: scatter (this rank's partial into every owner's receive buffer)
    -> barrier -> sum this rank's slots (+ bias, + residual) and store the
    token slice into every rank's output -> barrier.  Together an all-reduce;
    the data moves only in the library's peer stores.  The first barrier makes
    every partial visible before any rank sums; the second makes every slice
    visible before any rank reads its output, and keeps the next call from
    overwriting slots or outputs a slower rank still uses.

    ``recv`` holds the receive buffers (:func:`recv_buffer_numel` elements),
    ``out`` the ``[batch*seq, N]`` outputs.  ``w_shard`` is ``[N, k]``, this
    rank's columns of the unsharded weight.  ``scatter`` and ``reduce``
    default to the library's calls.
    """

    def __init__(self, w_shard: torch.Tensor, rank: int, tp: int, recv: PeerBuffers,
                 out: PeerBuffers, barrier: Callable, scatter: Optional[Callable] = None,
                 reduce: Optional[Callable] = None):
        self.w = w_shard.contiguous()
        self.rank, self.tp, self.recv, self.out = rank, tp, recv, out
        self.barrier = barrier
        self.scatter = scatter or tpl_row_linear_scatter
        self.reduce = reduce or tpl_reduce_slots_allgather

    def __call__(self, h_shard: torch.Tensor, batch: int, seq: int,
                 bias: Optional[torch.Tensor] = None, residual: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        """``h_shard`` ``[batch*seq, k]``; ``residual`` this rank's full
        ``[batch*seq, N]`` residual stream (it may be ``out.local``).  Returns
        ``out.local`` as ``[batch*seq, N]``, the full Y."""
        N = self.w.shape[0]
        sp_rows(batch, seq, self.tp)
        self.scatter(h_shard, self.w, batch, seq, self.rank, self.tp, self.recv.addrs,
                     stream=stream)
        self.barrier(stream)
        self.reduce(self.recv.local, self.tp, batch, seq, N, self.rank, self.out.addrs,
                    bias=bias, residual=residual, stream=stream)
        self.barrier(stream)
        return self.out.local.view(batch * seq, N)


class TPRankMLP:
    """Rank ``rank``'s share of the sequence-parallel TP MLP block over ``tp``
    GPUs (nanotron "MLP Module": activations ``[batch, seq // tp, hidden]`` per
    rank, gathered ahead of the column-parallel c_fc and reduce-scattered after
    the row-parallel c_proj; google-research residual section):

      RMSNorm of its token slice -> barrier -> c_fc + act over all tokens, each
      token tile read from the rank that owns it -> c_proj, partials scattered
      to the owner ranks -> barrier -> its slots summed with the residual, in
      place on its slice -> barrier.

    The first barrier makes every normalised slice visible before any rank
    reads it; the second every partial before any rank sums; the third keeps
    the next call from overwriting normalised slices or slots a slower rank
    still reads.  ``xn`` and ``recv`` are the peer-visible buffers
    (``[batch*seq/tp, hidden]`` and :func:`recv_buffer_numel` elements).
    ``w1_shard`` is ``[inter/tp, hidden]``, ``w2_shard`` ``[hidden, inter/tp]``.
    The ops default to the library's calls.
    """

    def __init__(self, w1_shard: torch.Tensor, w2_shard: torch.Tensor, rank: int, tp: int,
                 act: str, xn: PeerBuffers, recv: PeerBuffers, barrier: Callable,
                 scale: Optional[torch.Tensor] = None, centered: bool = False,
                 eps: float = 1e-6, ops: Optional[dict] = None):
        self.w1, self.w2 = w1_shard.contiguous(), w2_shard.contiguous()
        self.rank, self.tp, self.act = rank, tp, act
        self.xn, self.recv, self.barrier = xn, recv, barrier
        self.scale, self.centered, self.eps = scale, centered, eps
        self.part = tpl_partition_subparams([self.w1.shape[0]], 1, 1)
        ops = ops or {}
        self.rmsnorm = ops.get("rmsnorm", tpl_rmsnorm)
        self.column = ops.get("column", tpl_column_linear_gather)
        self.scatter = ops.get("scatter", tpl_row_linear_scatter)
        self.reduce = ops.get("reduce", tpl_reduce_slots)
        self.reduce_norm = ops.get("reduce_norm", tpl_reduce_slots_rmsnorm)
        self._h = None

    STEPS = ("rmsnorm", "barrier_xn", "column_gather", "row_scatter", "barrier_slots",
             "reduce_slots", "barrier_done")

    def __call__(self, x_slice: torch.Tensor, batch: int, seq: int, stream=None,
                 on_step: Optional[Callable] = None, normed: bool = False,
                 norm_next: Optional["TPRankMLP"] = None) -> torch.Tensor:
        """``x_slice`` ``[batch*seq/tp, hidden]``: this rank's tokens of the residual
        stream, updated in place to ``x + MLP(RMSNorm(x))``.  ``on_step(i)`` is
        called before step i of :attr:`STEPS` (e.g. to record a CUDA event).

        ``norm_next`` (the next layer, possibly this one again) makes the slot
        reduction also write RMSNorm of the updated slice, with that layer's
        scale, into that layer's ``xn`` (tpl_reduce_slots_rmsnorm); the next
        call then passes ``normed=True`` and skips its RMSNorm and the barrier
        after it: the barrier that ends this call already orders every rank's
        normalised slice before any rank's gather.  Every rank must pass the
        same flags (they decide which barriers run)."""
        H, tp = self.w2.shape[0], self.tp
        M = batch * seq
        sp_rows(batch, seq, tp)
        mark = on_step or (lambda i: None)
        if self._h is None or self._h.numel() < M * self.w1.shape[0]:
            self._h = torch.empty(M * self.w1.shape[0], dtype=x_slice.dtype,
                                  device=x_slice.device)
        mark(0)
        if not normed:
            self.rmsnorm(x_slice, self.scale, self.centered, self.eps, y=self.xn.local,
                         stream=stream)
        mark(1)
        if not normed:
            self.barrier(stream)
        mark(2)
        h = self.column(self.part, self.xn.addrs, batch, seq, self.w1, None, self.act,
                        y=self._h, stream=stream)
        mark(3)
        self.scatter(h.view(M, -1), self.w2, batch, seq, self.rank, tp, self.recv.addrs,
                     stream=stream)
        mark(4)
        self.barrier(stream)
        mark(5)
        if norm_next is None:
            self.reduce(self.recv.local, tp, H, None, x_slice, x_slice, stream=stream)
        else:
            self.reduce_norm(self.recv.local, tp, H, norm_next.xn.local, norm_next.scale,
                             norm_next.centered, norm_next.eps, None, x_slice, x_slice,
                             stream=stream)
        mark(6)
        self.barrier(stream)
        return x_slice


class TPLMHeadRank:
    """Rank ``rank``'s share of the decode LM head over ``tp`` GPUs (Tenstorrent
    LMHead1D: every device computes its vocab slice; the candidates are combined
    at the end): the argmax candidates of its slice, all-gathered (8 bytes per
    row per rank), merged into global ids.

    ``w_slice`` is rows ``rank * shard .. (rank+1) * shard`` of W, with
    ``shard = ceil(V / tp)``.  ``local_argmax``, ``gather`` and ``merge``
    default to the library's calls and the process group's all-gather.
    """

    def __init__(self, w_slice: torch.Tensor, rank: int, tp: int, shard: int, group=None,
                 local_argmax: Optional[Callable] = None, gather: Optional[Callable] = None,
                 merge: Optional[Callable] = None):
        self.w = w_slice.contiguous()
        self.rank, self.tp, self.shard, self.group = rank, tp, shard, group
        self._own_argmax = local_argmax is None
        self.local_argmax = local_argmax or self._local_argmax
        self.gather = gather or self._gather
        self.merge = merge or (lambda m, i, stride, stream=None:
                               tpl_argmax_merge(m, i, stride, stream=stream))
        self._ws = None

    def _local_argmax(self, x, stream=None):
        B = x.shape[0]
        need = tpl_lmhead_workspace_size(B, self.w.shape[0], 1, 1)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
        _, m, i = tpl_lmhead_argmax(x, self.w, 1, 1, self._ws, stream=stream)
        return m[0], i[0]

    def _gather(self, t: torch.Tensor, stream=None) -> torch.Tensor:
        """``[tp, ...]``: every rank's ``t``, in rank order."""
        import torch.distributed as dist
        parts = [torch.empty_like(t) for _ in range(self.tp)]
        if stream is None:
            dist.all_gather(parts, t, group=self.group)
            return torch.stack(parts)
        with torch.cuda.stream(stream):
            dist.all_gather(parts, t, group=self.group)
            return torch.stack(parts)

    def __call__(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """``x`` ``[B, K]`` (the same on every rank).  Returns global ids ``[B]``.

        With the library's local argmax, the call ends by reading the device
        status (which waits for the stream: a decode step needs its ids on the
        host anyway).  A kernel that gave up waiting leaves its workspace
        stale, so the workspace is cleared and the call raises TplError; the
        next call starts clean."""
        m, i = self.local_argmax(x, stream=stream)
        ids = self.merge(self.gather(m, stream=stream), self.gather(i, stream=stream),
                         self.shard, stream=stream)
        if self._own_argmax:
            code = tpl_get_device_status(stream)
            if code != 0:
                if self._ws is not None:
                    self._ws.zero_()
                raise TplError(code, "TPLMHeadRank")
        return ids
