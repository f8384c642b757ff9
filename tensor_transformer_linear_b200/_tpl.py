"""ctypes binding of libtpl.so: argument marshalling only.

Every function here has the name of the C entry point it calls and does
nothing but check that torch tensors are CUDA tensors of the right dtype and
shape, pass their data pointers and the current stream, and turn a non-zero
status into :class:`TplError`.  Output tensors the caller does not pass are
allocated with torch (device memory is torch's job).  There is no CPU path: a
CPU tensor, or a missing ``libtpl.so``, raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtpl.so")

TPL_MAX_TP = 64
TPL_MAX_SUB = 8

STATUS = {0: "TPL_OK", 1: "TPL_ERR_NULL", 2: "TPL_ERR_SHAPE", 3: "TPL_ERR_INDIVISIBLE",
          4: "TPL_ERR_DTYPE", 5: "TPL_ERR_ALIGN", 6: "TPL_ERR_CUDA", 7: "TPL_ERR_TIMEOUT",
          8: "TPL_ERR_UNSUPPORTED"}
ACT = {"none": 0, None: 0, "gelu_erf": 1, "gelu_tanh": 2}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}

EXPORTED = ("tpl_partition_subparams", "tpl_column_linear", "tpl_row_linear_reduce",
            "tpl_rmsnorm", "tpl_lmhead_workspace_size", "tpl_lmhead_argmax",
            "tpl_get_device_status", "tpl_status_string", "tpl_launch_count",
            "tpl_lmhead_argmax_static", "tpl_row_linear_reduce_scatter",
            "tpl_column_linear_allgather", "tpl_swiglu_column_linear", "tpl_embedding_lookup",
            "tpl_selftest_wait_timeout", "tpl_row_linear_scatter", "tpl_reduce_slots",
            "tpl_argmax_merge", "tpl_column_linear_gather", "tpl_reduce_slots_allgather",
            "tpl_column_linear_rmsnorm_workspace_size", "tpl_column_linear_rmsnorm",
            "tpl_fold_norm_scale", "tpl_trace_set", "tpl_reduce_slots_rmsnorm",
            "tpl_tp_mlp_fp32")


class TplError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.name = STATUS.get(code, str(code))
        super().__init__(f"{where}: {self.name}")


class Partition(ctypes.Structure):
    _fields_ = [("tp_size", ctypes.c_int32), ("n_sub", ctypes.c_int32),
                ("logical_out", ctypes.c_int64),
                ("width", (ctypes.c_int64 * TPL_MAX_SUB) * TPL_MAX_TP),
                ("src_off", (ctypes.c_int64 * TPL_MAX_SUB) * TPL_MAX_TP),
                ("dst_off", (ctypes.c_int64 * TPL_MAX_SUB) * TPL_MAX_TP),
                ("shard_width", ctypes.c_int64 * TPL_MAX_TP),
                ("shard_base", ctypes.c_int64 * TPL_MAX_TP)]

    def as_lists(self):
        tp, ns = self.tp_size, self.n_sub
        return dict(width=[[self.width[r][j] for j in range(ns)] for r in range(tp)],
                    src_off=[[self.src_off[r][j] for j in range(ns)] for r in range(tp)],
                    dst_off=[[self.dst_off[r][j] for j in range(ns)] for r in range(tp)],
                    shard_width=[self.shard_width[r] for r in range(tp)],
                    shard_base=[self.shard_base[r] for r in range(tp)])


_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m tensor_transformer_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.tpl_partition_subparams.argtypes = [ctypes.POINTER(i64), i32, i32, i64,
                                              ctypes.POINTER(Partition)]
        L.tpl_column_linear.argtypes = [ctypes.POINTER(Partition), vp, i64, i64, vp, vp, i32, i32,
                                        vp, vp]
        L.tpl_row_linear_reduce.argtypes = [vp, ctypes.POINTER(i64), i32, i64, i64, vp, vp, vp,
                                            i32, vp, vp, vp]
        L.tpl_rmsnorm.argtypes = [vp, i64, i64, vp, i32, ctypes.c_float, i32, vp, vp]
        L.tpl_lmhead_workspace_size.argtypes = [i64, i64, i32, i32, ctypes.POINTER(sz)]
        L.tpl_lmhead_argmax.argtypes = [vp, i64, i64, vp, i64, i32, i32, vp, vp, vp, vp, vp, sz,
                                        vp]
        L.tpl_lmhead_argmax_static.argtypes = [vp, i64, i64, vp, i64, i32, i32, vp, vp, vp, vp,
                                               vp]
        L.tpl_row_linear_reduce_scatter.argtypes = [vp, ctypes.POINTER(i64), i32, i64, i64, i64,
                                                    vp, vp, vp, i32, vp, vp]
        L.tpl_column_linear_allgather.argtypes = [ctypes.POINTER(Partition), vp, i64, i64, i64,
                                                  vp, vp, i32, i32, vp, vp]
        L.tpl_swiglu_column_linear.argtypes = [vp, i64, i64, vp, i64, i32, i32, vp, vp]
        L.tpl_embedding_lookup.argtypes = [vp, i64, vp, i64, i64, i32, i32, vp, vp]
        L.tpl_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp, vp]
        L.tpl_row_linear_scatter.argtypes = [vp, i64, i64, i64, i64, vp, i32, i32,
                                             ctypes.POINTER(vp), vp]
        L.tpl_reduce_slots.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp]
        L.tpl_reduce_slots_rmsnorm.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp, i32,
                                               ctypes.c_float, vp, vp]
        L.tpl_reduce_slots_allgather.argtypes = [vp, i32, i64, i64, i64, vp, vp, i32,
                                                 ctypes.POINTER(vp), vp]
        L.tpl_argmax_merge.argtypes = [vp, vp, i32, i64, i64, vp, vp]
        L.tpl_column_linear_gather.argtypes = [ctypes.POINTER(Partition), ctypes.POINTER(vp), i32,
                                               i64, i64, i64, vp, vp, i32, vp, vp]
        L.tpl_column_linear_rmsnorm_workspace_size.argtypes = [i64, ctypes.POINTER(sz)]
        L.tpl_column_linear_rmsnorm.argtypes = [ctypes.POINTER(Partition), vp, i64, i64, vp, vp,
                                                ctypes.c_float, i32, vp, vp, sz, vp]
        L.tpl_fold_norm_scale.argtypes = [vp, i64, i64, vp, i32, vp, vp]
        L.tpl_trace_set.argtypes = [vp, i64]
        L.tpl_tp_mlp_fp32.argtypes = [vp, i64, i64, vp, vp, i64, i32, i32, vp, vp, vp, vp, vp]
        L.tpl_get_device_status.argtypes = [vp]
        L.tpl_status_string.argtypes = [i32]
        L.tpl_status_string.restype = ctypes.c_char_p
        L.tpl_launch_count.restype = ctypes.c_uint64
        for name in EXPORTED:
            if name not in ("tpl_status_string", "tpl_launch_count"):
                getattr(L, name).restype = i32
        _lib = L
    return _lib


def _check(code: int, where: str):
    if code != 0:
        raise TplError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (this library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


# ---------------------------------------------------------------- entry points

def tpl_partition_subparams(sub_sizes: Sequence[int], tp: int, align: int = 1) -> Partition:
    arr = (ctypes.c_int64 * max(1, len(sub_sizes)))(*[int(s) for s in sub_sizes])
    p = Partition()
    _check(lib().tpl_partition_subparams(arr, len(sub_sizes), int(tp), int(align),
                                         ctypes.byref(p)), "tpl_partition_subparams")
    return p


def _ws(workspace: Optional[torch.Tensor]):
    _cuda(workspace, "workspace")
    return _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size())


def tpl_column_linear(p: Partition, x: torch.Tensor, w: torch.Tensor,
                      bias: Optional[torch.Tensor] = None, act: str = "none",
                      y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Returns y holding every rank's shard (rank r: ``[M, shard_width[r]]`` at M*shard_base[r])."""
    _cuda(x, "x")
    dt = x.dtype
    _cuda(w, "w", dt)
    if bias is not None:
        _cuda(bias, "bias", dt)
    M, K = x.shape[0] if x.dim() == 2 else x.numel() // x.shape[-1], x.shape[-1]
    if y is None:
        y = torch.empty(M * p.logical_out, dtype=dt, device=x.device)
    _cuda(y, "y", dt)
    if y.numel() < M * p.logical_out or w.numel() != p.logical_out * K:
        raise ValueError("y or w has the wrong size")
    if bias is not None and bias.numel() != p.logical_out:
        raise ValueError("bias size does not match the partition's output size")
    _check(lib().tpl_column_linear(ctypes.byref(p), _ptr(x), M, K, _ptr(w), _ptr(bias),
                                   DTYPE[dt], ACT[act], _ptr(y), _stream(stream)),
           "tpl_column_linear")
    return y


def tpl_column_linear_rmsnorm_workspace_size(M: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tpl_column_linear_rmsnorm_workspace_size(int(M), ctypes.byref(n)),
           "tpl_column_linear_rmsnorm_workspace_size")
    return int(n.value)


def rmsnorm_linear_workspace(M: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for tpl_column_linear_rmsnorm with up to M rows
    (reusable across calls on one stream)."""
    with torch.cuda.device(device):
        n = tpl_column_linear_rmsnorm_workspace_size(M)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def tpl_fold_norm_scale(w: torch.Tensor, scale: torch.Tensor, centered: bool = False,
                        out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``w[n][k] * g[k]`` in bf16, g = 1 + scale (centred) or scale: an RMSNorm's
    scale folded into the weight of the column-parallel linear that follows it."""
    _cuda(w, "w", torch.bfloat16)
    _cuda(scale, "scale", torch.float32)
    K = w.shape[-1]
    if scale.numel() != K:
        raise ValueError("scale must be [K]")
    if out is None:
        out = torch.empty_like(w)
    _cuda(out, "out", torch.bfloat16)
    _check(lib().tpl_fold_norm_scale(_ptr(w), w.numel() // K, K, _ptr(scale), int(bool(centered)),
                                     _ptr(out), _stream(stream)), "tpl_fold_norm_scale")
    return out


def tpl_column_linear_rmsnorm(p: Partition, x: torch.Tensor, w: torch.Tensor,
                              bias: Optional[torch.Tensor], eps: float, act: str,
                              workspace: torch.Tensor, y: Optional[torch.Tensor] = None,
                              stream=None) -> torch.Tensor:
    """Column-parallel linear of RMSNorm(x) with the norm fused in: ``w`` is the
    weight with the norm's scale folded in (:func:`tpl_fold_norm_scale`), x the
    raw activations; ``workspace`` from :func:`rmsnorm_linear_workspace`."""
    _cuda(x, "x", torch.bfloat16)
    _cuda(w, "w", torch.bfloat16)
    if bias is not None:
        _cuda(bias, "bias", torch.bfloat16)
    M, K = x.numel() // x.shape[-1], x.shape[-1]
    if y is None:
        y = torch.empty(M * p.logical_out, dtype=torch.bfloat16, device=x.device)
    _cuda(y, "y", torch.bfloat16)
    if y.numel() < M * p.logical_out or w.numel() != p.logical_out * K:
        raise ValueError("y or w has the wrong size")
    _check(lib().tpl_column_linear_rmsnorm(ctypes.byref(p), _ptr(x), M, K, _ptr(w), _ptr(bias),
                                           float(eps), ACT[act], _ptr(y), *_ws(workspace),
                                           _stream(stream)), "tpl_column_linear_rmsnorm")
    return y


def tpl_row_linear_reduce(h: torch.Tensor, k_w: Sequence[int], M: int, w: torch.Tensor,
                          bias: Optional[torch.Tensor] = None,
                          residual: Optional[torch.Tensor] = None,
                          y: Optional[torch.Tensor] = None,
                          partials: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``Y = sum_r H_r W2_r^T (+ bias) (+ residual)``; h and w are rank-major packed blocks."""
    _cuda(h, "h")
    dt = h.dtype
    _cuda(w, "w", dt)
    tp = len(k_w)
    ktot = sum(int(k) for k in k_w)
    if h.numel() != M * ktot or w.numel() % ktot != 0:
        raise ValueError("h or w has the wrong size")
    N = w.numel() // ktot
    if y is None:
        y = torch.empty((M, N), dtype=dt, device=h.device)
    _cuda(y, "y", dt)
    if residual is not None:
        _cuda(residual, "residual", dt)
    if bias is not None:
        _cuda(bias, "bias", dt)
    if partials is not None:
        _cuda(partials, "partials", torch.float32)
        if partials.numel() != tp * M * N:
            raise ValueError("partials must hold tp * M * N floats")
    kw = (ctypes.c_int64 * tp)(*[int(k) for k in k_w])
    _check(lib().tpl_row_linear_reduce(_ptr(h), kw, tp, int(M), int(N), _ptr(w), _ptr(bias),
                                       _ptr(residual), DTYPE[dt], _ptr(y), _ptr(partials),
                                       _stream(stream)), "tpl_row_linear_reduce")
    return y


def tpl_rmsnorm(x: torch.Tensor, scale: Optional[torch.Tensor] = None, centered: bool = False,
                eps: float = 1e-6, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _cuda(x, "x")
    H = x.shape[-1]
    M = x.numel() // H
    if y is None:
        y = torch.empty_like(x)
    _cuda(y, "y", x.dtype)
    if scale is not None:
        _cuda(scale, "scale", torch.float32)
        if scale.numel() != H:
            raise ValueError("scale must have H elements")
    _check(lib().tpl_rmsnorm(_ptr(x), M, H, _ptr(scale), 1 if centered else 0,
                             ctypes.c_float(eps), DTYPE[x.dtype], _ptr(y), _stream(stream)),
           "tpl_rmsnorm")
    return y


def tpl_lmhead_workspace_size(B: int, V: int, tp: int, n_chunks: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tpl_lmhead_workspace_size(int(B), int(V), int(tp), int(n_chunks),
                                           ctypes.byref(n)), "tpl_lmhead_workspace_size")
    return n.value


def lmhead_workspace(B: int, V: int, tp: int, n_chunks: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for tpl_lmhead_argmax (reusable across calls)."""
    n = tpl_lmhead_workspace_size(B, V, tp, n_chunks)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def tpl_lmhead_argmax(x: torch.Tensor, w: torch.Tensor, tp: int, n_chunks: int,
                      workspace: torch.Tensor, logits: Optional[torch.Tensor] = None,
                      ids: Optional[torch.Tensor] = None,
                      shard_max: Optional[torch.Tensor] = None,
                      shard_idx: Optional[torch.Tensor] = None, stream=None):
    """Returns ``(ids [B], shard_max [tp, B], shard_idx [tp, B])``; fills ``logits`` if given."""
    _cuda(x, "x", torch.bfloat16)
    _cuda(w, "w", torch.bfloat16)
    _cuda(workspace, "workspace")
    B, K = x.shape
    V = w.shape[0]
    dev = x.device
    if ids is None:
        ids = torch.empty(B, dtype=torch.int32, device=dev)
    if shard_max is None:
        shard_max = torch.empty((tp, B), dtype=torch.float32, device=dev)
    if shard_idx is None:
        shard_idx = torch.empty((tp, B), dtype=torch.int32, device=dev)
    if logits is not None:
        _cuda(logits, "logits", torch.float32)
        if logits.numel() != B * V:
            raise ValueError("logits must hold B * V floats")
    _check(lib().tpl_lmhead_argmax(_ptr(x), B, K, _ptr(w), V, int(tp), int(n_chunks),
                                   _ptr(logits), _ptr(shard_max), _ptr(shard_idx), _ptr(ids),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)), "tpl_lmhead_argmax")
    return ids, shard_max, shard_idx


def tpl_lmhead_argmax_static(x: torch.Tensor, w: torch.Tensor, tp: int, n_chunks: int,
                             logits: Optional[torch.Tensor] = None,
                             ids: Optional[torch.Tensor] = None,
                             shard_max: Optional[torch.Tensor] = None,
                             shard_idx: Optional[torch.Tensor] = None, stream=None):
    """tpl_lmhead_argmax without a workspace: the library's own fixed scratch is used.

    For callers that cannot allocate device memory.  Calls that overlap on the
    GPU share that scratch and race; order them on one stream.
    """
    _cuda(x, "x", torch.bfloat16)
    _cuda(w, "w", torch.bfloat16)
    B, K = x.shape
    V = w.shape[0]
    dev = x.device
    if ids is None:
        ids = torch.empty(B, dtype=torch.int32, device=dev)
    if shard_max is None:
        shard_max = torch.empty((tp, B), dtype=torch.float32, device=dev)
    if shard_idx is None:
        shard_idx = torch.empty((tp, B), dtype=torch.int32, device=dev)
    if logits is not None:
        _cuda(logits, "logits", torch.float32)
        if logits.numel() != B * V:
            raise ValueError("logits must hold B * V floats")
    _check(lib().tpl_lmhead_argmax_static(_ptr(x), B, K, _ptr(w), V, int(tp), int(n_chunks),
                                          _ptr(logits), _ptr(shard_max), _ptr(shard_idx),
                                          _ptr(ids), _stream(stream)),
           "tpl_lmhead_argmax_static")
    return ids, shard_max, shard_idx


def tpl_row_linear_reduce_scatter(h: torch.Tensor, k_w: Sequence[int], batch: int, seq: int,
                                  w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                                  residual: Optional[torch.Tensor] = None,
                                  y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Row-parallel linear; the summed output is returned rank-major ``[tp, batch, seq/tp, N]``."""
    _cuda(h, "h")
    dt = h.dtype
    _cuda(w, "w", dt)
    tp = len(k_w)
    ktot = sum(int(k) for k in k_w)
    M = batch * seq
    if h.numel() != M * ktot or w.numel() % ktot != 0:
        raise ValueError("h or w has the wrong size")
    N = w.numel() // ktot
    if y is None:
        y = torch.empty((tp, batch, seq // tp, N), dtype=dt, device=h.device)
    _cuda(y, "y", dt)
    if residual is not None:
        _cuda(residual, "residual", dt)
    if bias is not None:
        _cuda(bias, "bias", dt)
    kw = (ctypes.c_int64 * tp)(*[int(k) for k in k_w])
    _check(lib().tpl_row_linear_reduce_scatter(_ptr(h), kw, tp, int(batch), int(seq), int(N),
                                               _ptr(w), _ptr(bias), _ptr(residual), DTYPE[dt],
                                               _ptr(y), _stream(stream)),
           "tpl_row_linear_reduce_scatter")
    return y


def tpl_column_linear_allgather(p: Partition, x_sp: torch.Tensor, batch: int, seq: int,
                                w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                                act: str = "none", y: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """Column-parallel linear reading sequence-sharded, rank-major activations."""
    _cuda(x_sp, "x")
    dt = x_sp.dtype
    _cuda(w, "w", dt)
    K = x_sp.shape[-1]
    M = batch * seq
    if x_sp.numel() != M * K or w.numel() != p.logical_out * K:
        raise ValueError("x or w has the wrong size")
    if bias is not None:
        _cuda(bias, "bias", dt)
    if y is None:
        y = torch.empty(M * p.logical_out, dtype=dt, device=x_sp.device)
    _cuda(y, "y", dt)
    _check(lib().tpl_column_linear_allgather(ctypes.byref(p), _ptr(x_sp), int(batch), int(seq),
                                             int(K), _ptr(w), _ptr(bias), DTYPE[dt], ACT[act],
                                             _ptr(y), _stream(stream)),
           "tpl_column_linear_allgather")
    return y


def tpl_swiglu_column_linear(x: torch.Tensor, w: torch.Tensor, F: int, tp: int,
                             h: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Fused SwiGLU column projection; rank r's ``[M, F_r]`` block at M * sum(F_q, q < r)."""
    _cuda(x, "x")
    dt = x.dtype
    _cuda(w, "w", dt)
    M, K = x.shape
    if w.numel() != 2 * F * K:
        raise ValueError("w must be [2F, K]")
    if h is None:
        h = torch.empty(M * F, dtype=dt, device=x.device)
    _cuda(h, "h", dt)
    _check(lib().tpl_swiglu_column_linear(_ptr(x), int(M), int(K), _ptr(w), int(F), int(tp),
                                          DTYPE[dt], _ptr(h), _stream(stream)),
           "tpl_swiglu_column_linear")
    return h


def tpl_embedding_lookup(ids: torch.Tensor, table: torch.Tensor, tp: int,
                         out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Vocab-sharded embedding: ``[n, H]`` rows of ``table``, zeros for ids outside [0, V)."""
    _cuda(ids, "ids", torch.int32)
    _cuda(table, "table")
    V, H = table.shape
    n = ids.numel()
    if out is None:
        out = torch.empty((n, H), dtype=table.dtype, device=table.device)
    _cuda(out, "out", table.dtype)
    _check(lib().tpl_embedding_lookup(_ptr(ids), int(n), _ptr(table), int(V), int(H), int(tp),
                                      DTYPE[table.dtype], _ptr(out), _stream(stream)),
           "tpl_embedding_lookup")
    return out


def _addresses(bufs: Sequence, name: str, dtype=torch.bfloat16):
    """Device addresses of CUDA tensors, or integers given as addresses (mapped peer buffers)."""
    out = []
    for q, b in enumerate(bufs):
        if isinstance(b, torch.Tensor):
            _cuda(b, f"{name}[{q}]", dtype)
            out.append(b.data_ptr())
        else:
            out.append(int(b))
    return (ctypes.c_void_p * len(out))(*out)


def tpl_column_linear_gather(p: Partition, peer_x: Sequence, batch: int, seq: int,
                             w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                             act: str = "none", y: Optional[torch.Tensor] = None,
                             stream=None) -> torch.Tensor:
    """This rank's column shard over every rank's token slice ``peer_x[q]``
    (``[batch, seq // tp, K]`` bf16, a CUDA tensor or a mapped peer address)."""
    _cuda(w, "w", torch.bfloat16)
    if bias is not None:
        _cuda(bias, "bias", torch.bfloat16)
    tp = len(peer_x)
    K = w.shape[-1]
    M = int(batch) * int(seq)
    for q, b in enumerate(peer_x):
        if isinstance(b, torch.Tensor) and b.numel() != M // tp * K:
            raise ValueError(f"peer_x[{q}] must be [batch, seq // tp, K]")
    if w.numel() != p.logical_out * K:
        raise ValueError("w must be [logical_out, K]")
    if bias is not None and bias.numel() != p.logical_out:
        raise ValueError("bias must be [logical_out]")
    if y is None:
        y = torch.empty(M * p.logical_out, dtype=torch.bfloat16, device=w.device)
    _cuda(y, "y", torch.bfloat16)
    if y.numel() < M * p.logical_out:
        raise ValueError("y must hold batch * seq * logical_out elements")
    _check(lib().tpl_column_linear_gather(ctypes.byref(p), _addresses(peer_x, "peer_x"),
                                          int(tp), int(batch), int(seq), int(K), _ptr(w),
                                          _ptr(bias), ACT[act], _ptr(y), _stream(stream)),
           "tpl_column_linear_gather")
    return y


def tpl_row_linear_scatter(h: torch.Tensor, w: torch.Tensor, batch: int, seq: int, rank: int,
                           tp: int, peers: Sequence, stream=None) -> None:
    """This rank's row-parallel shard, written into every owner rank's receive buffer.

    ``peers[q]`` is rank q's receive buffer ``[tp][batch][seq // tp][N]`` bf16:
    a CUDA tensor, or the integer device address of a buffer mapped from
    another GPU (see include/tpl.h).
    """
    _cuda(h, "h", torch.bfloat16)
    _cuda(w, "w", torch.bfloat16)
    M, K = int(batch) * int(seq), h.shape[-1]
    if h.numel() != M * K or w.numel() % K != 0:
        raise ValueError("h must be [batch * seq, K] and w [N, K]")
    N = w.numel() // K
    if len(peers) != tp:
        raise ValueError("peers must hold one receive buffer per rank")
    addr = []
    for q, p in enumerate(peers):
        if isinstance(p, torch.Tensor):
            _cuda(p, f"peers[{q}]", torch.bfloat16)
            if p.numel() < M * N:
                raise ValueError(f"peers[{q}] is smaller than [tp][batch][seq // tp][N]")
            addr.append(p.data_ptr())
        else:
            addr.append(int(p))
    arr = (ctypes.c_void_p * tp)(*addr)
    _check(lib().tpl_row_linear_scatter(_ptr(h), int(K), int(batch), int(seq), int(N), _ptr(w),
                                        int(rank), int(tp), arr, _stream(stream)),
           "tpl_row_linear_scatter")


def tpl_reduce_slots(recv: torch.Tensor, tp: int, N: int, bias: Optional[torch.Tensor] = None,
                     residual: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """``y = sum of the tp slots of recv (+ bias) (+ residual)``: this rank's token slice."""
    _cuda(recv, "recv", torch.bfloat16)
    if recv.numel() % (tp * N) != 0:
        raise ValueError("recv must be [tp][rows][N]")
    rows = recv.numel() // (tp * N)
    if y is None:
        y = torch.empty((rows, N), dtype=torch.bfloat16, device=recv.device)
    _cuda(y, "y", torch.bfloat16)
    if bias is not None:
        _cuda(bias, "bias", torch.bfloat16)
        if bias.numel() != N:
            raise ValueError("bias must be [N]")
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
        if residual.numel() != rows * N:
            raise ValueError("residual must be [rows][N]")
    if y.numel() != rows * N:
        raise ValueError("y must be [rows][N]")
    _check(lib().tpl_reduce_slots(_ptr(recv), int(tp), int(rows), int(N), _ptr(bias),
                                  _ptr(residual), _ptr(y), _stream(stream)), "tpl_reduce_slots")
    return y


def tpl_tp_mlp_fp32(x: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor, tp: int, act: str,
                    b1: Optional[torch.Tensor] = None, b2: Optional[torch.Tensor] = None,
                    residual: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """The fp32 TP MLP block in one launch: ``act(x W1^T + b1) W2^T + b2 (+ residual)``;
    ``w2`` in the per-rank packed layout of :func:`pack_row_weight` (equal widths).
    Raises TplError TPL_ERR_UNSUPPORTED for shapes the fused kernel does not take."""
    _cuda(x, "x", torch.float32)
    _cuda(w1, "w1", torch.float32)
    _cuda(w2, "w2", torch.float32)
    I, H = w1.shape
    M = x.numel() // H
    if x.shape[-1] != H or w2.numel() != H * I:
        raise ValueError("x must be [M][H], w1 [I][H] and w2 hold H * I elements")
    for t, n, name in ((b1, I, "b1"), (b2, H, "b2")):
        if t is not None:
            _cuda(t, name, torch.float32)
            if t.numel() != n:
                raise ValueError(f"{name} must hold {n} elements")
    if residual is not None:
        _cuda(residual, "residual", torch.float32)
        if residual.numel() != M * H:
            raise ValueError("residual must be [M][H]")
    if y is None:
        y = torch.empty((M, H), dtype=torch.float32, device=x.device)
    _cuda(y, "y", torch.float32)
    if y.numel() != M * H:
        raise ValueError("y must be [M][H]")
    _check(lib().tpl_tp_mlp_fp32(_ptr(x), int(M), int(H), _ptr(w1), _ptr(b1), int(I), int(tp),
                                 ACT[act], _ptr(w2), _ptr(b2), _ptr(residual), _ptr(y),
                                 _stream(stream)), "tpl_tp_mlp_fp32")
    return y


def tpl_reduce_slots_rmsnorm(recv: torch.Tensor, tp: int, N: int, xn: torch.Tensor,
                             scale: Optional[torch.Tensor] = None, centered: bool = False,
                             eps: float = 1e-6, bias: Optional[torch.Tensor] = None,
                             residual: Optional[torch.Tensor] = None,
                             y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """:func:`tpl_reduce_slots` plus ``xn = RMSNorm(y)`` (fp32 ``scale``, centred or
    not) written in the same pass: the next layer's normalised input."""
    _cuda(recv, "recv", torch.bfloat16)
    if recv.numel() % (tp * N) != 0:
        raise ValueError("recv must be [tp][rows][N]")
    rows = recv.numel() // (tp * N)
    if y is None:
        y = torch.empty((rows, N), dtype=torch.bfloat16, device=recv.device)
    _cuda(y, "y", torch.bfloat16)
    _cuda(xn, "xn", torch.bfloat16)
    if bias is not None:
        _cuda(bias, "bias", torch.bfloat16)
        if bias.numel() != N:
            raise ValueError("bias must be [N]")
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
        if residual.numel() != rows * N:
            raise ValueError("residual must be [rows][N]")
    if scale is not None:
        _cuda(scale, "scale", torch.float32)
        if scale.numel() != N:
            raise ValueError("scale must be [N]")
    if y.numel() != rows * N or xn.numel() != rows * N:
        raise ValueError("y and xn must be [rows][N]")
    _check(lib().tpl_reduce_slots_rmsnorm(_ptr(recv), int(tp), int(rows), int(N), _ptr(bias),
                                          _ptr(residual), _ptr(y), _ptr(scale), int(bool(centered)),
                                          float(eps), _ptr(xn), _stream(stream)),
           "tpl_reduce_slots_rmsnorm")
    return y


def tpl_reduce_slots_allgather(recv: torch.Tensor, tp: int, batch: int, seq: int, N: int,
                               rank: int, peers_y: Sequence,
                               bias: Optional[torch.Tensor] = None,
                               residual: Optional[torch.Tensor] = None, stream=None) -> None:
    """This rank's token slice of ``sum of the tp slots of recv (+ bias)
    (+ residual)``, stored at its rows of every rank's full ``[batch * seq, N]``
    output ``peers_y[q]`` (a CUDA tensor, or a mapped peer address); see
    include/tpl.h.  ``residual`` is this rank's full ``[batch * seq, N]``
    residual stream and may be ``peers_y[rank]`` itself."""
    _cuda(recv, "recv", torch.bfloat16)
    M = int(batch) * int(seq)
    if len(peers_y) != tp:
        raise ValueError("peers_y must hold one output buffer per rank")
    if recv.numel() != M * N:
        raise ValueError("recv must be [tp][batch][seq // tp][N]")
    if bias is not None:
        _cuda(bias, "bias", torch.bfloat16)
        if bias.numel() != N:
            raise ValueError("bias must be [N]")
    if residual is not None:
        _cuda(residual, "residual", torch.bfloat16)
        if residual.numel() != M * N:
            raise ValueError("residual must be [batch * seq][N]")
    for q, t in enumerate(peers_y):
        if isinstance(t, torch.Tensor) and t.numel() < M * N:
            raise ValueError(f"peers_y[{q}] is smaller than [batch * seq][N]")
    _check(lib().tpl_reduce_slots_allgather(_ptr(recv), int(tp), int(batch), int(seq), int(N),
                                            _ptr(bias), _ptr(residual), int(rank),
                                            _addresses(peers_y, "peers_y"), _stream(stream)),
           "tpl_reduce_slots_allgather")


def tpl_argmax_merge(shard_max: torch.Tensor, shard_idx: torch.Tensor, id_stride: int,
                     ids: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Global argmax over ranks from the gathered ``[tp][B]`` per-rank LM-head outputs."""
    _cuda(shard_max, "shard_max", torch.float32)
    _cuda(shard_idx, "shard_idx", torch.int32)
    tp, B = shard_max.shape
    if shard_idx.shape != shard_max.shape:
        raise ValueError("shard_idx must match shard_max")
    if ids is None:
        ids = torch.empty(B, dtype=torch.int32, device=shard_max.device)
    _cuda(ids, "ids", torch.int32)
    if ids.numel() < B:
        raise ValueError("ids must hold B elements")
    _check(lib().tpl_argmax_merge(_ptr(shard_max), _ptr(shard_idx), int(tp), int(B),
                                  int(id_stride), _ptr(ids), _stream(stream)), "tpl_argmax_merge")
    return ids


def tpl_selftest_wait_timeout(limit_ns: int, waited_us: Optional[torch.Tensor] = None,
                              stream=None) -> None:
    """Run the bounded-wait failure path once (see include/tpl.h)."""
    if waited_us is not None:
        _cuda(waited_us, "waited_us", torch.int32)
    _check(lib().tpl_selftest_wait_timeout(int(limit_ns), _ptr(waited_us), _stream(stream)),
           "tpl_selftest_wait_timeout")


def tpl_get_device_status(stream=None) -> int:
    return lib().tpl_get_device_status(_stream(stream))


def tpl_status_string(code: int) -> str:
    return lib().tpl_status_string(int(code)).decode()


def tpl_launch_count() -> int:
    return int(lib().tpl_launch_count())


TRACE_HEADER_BYTES = 16
TRACE_RECORD_BYTES = 32
TRACE_KINDS = {1: "gemm", 2: "gemm_pair", 3: "lmhead"}


class Trace:
    """A trace buffer for tpl_trace_set: per-CTA timing records of the GEMM and
    LM-head kernels (launch number, kind, CTA, %globaltimer at start and end,
    SM cycles).  ``with Trace(capacity, device) as t: ...`` installs it on the
    current device for the block and removes it after; ``t.records()`` reads
    them back, ``t.launches()`` groups them per launch."""

    def __init__(self, capacity: int, device="cuda"):
        import torch
        self.capacity = int(capacity)
        n = (TRACE_HEADER_BYTES + TRACE_RECORD_BYTES * self.capacity) // 8
        self.buf = torch.zeros(n, dtype=torch.int64, device=device)

    def __enter__(self):
        _check(lib().tpl_trace_set(self.buf.data_ptr(), self.capacity), "tpl_trace_set")
        return self

    def __exit__(self, *exc):
        _check(lib().tpl_trace_set(None, 0), "tpl_trace_set")
        return False

    def records(self):
        """[(seq, kind, cta, t0_ns, t1_ns, cycles)] in the order the CTAs finished."""
        import numpy as np
        raw = self.buf.cpu().numpy()
        count = int(raw[:2].view(np.uint32)[0])
        rec = raw[TRACE_HEADER_BYTES // 8:].view(np.uint64).reshape(-1, 4)[:min(count, self.capacity)]
        out = []
        for w0, t0, t1, cyc in rec.tolist():
            out.append((w0 & 0xFFFFFFFF, (w0 >> 32) & 0xFFFF, w0 >> 48, t0, t1, cyc))
        return out

    def dropped(self) -> int:
        import numpy as np
        count = int(self.buf[:2].cpu().numpy().view(np.uint32)[0])
        return max(0, count - self.capacity)

    def launches(self):
        """Per launch, in launch order: {seq, kind, ctas, span_us (first CTA start
        to last CTA end), cta_us (median CTA duration), sm_mhz (median over CTAs
        of cycles / duration)}."""
        import statistics
        by = {}
        for seq, kind, cta, t0, t1, cyc in self.records():
            by.setdefault(seq, []).append((kind, t0, t1, cyc))
        out = []
        for seq in sorted(by):
            r = by[seq]
            dur = [t1 - t0 for _, t0, t1, _ in r]
            mhz = [c / (t1 - t0) * 1e3 for _, t0, t1, c in r if t1 > t0]
            out.append({"seq": seq, "kind": TRACE_KINDS.get(r[0][0], str(r[0][0])),
                        "ctas": len(r),
                        "span_us": (max(x[2] for x in r) - min(x[1] for x in r)) / 1e3,
                        "cta_us": statistics.median(dur) / 1e3,
                        "sm_mhz": statistics.median(mhz) if mhz else None})
        return out
