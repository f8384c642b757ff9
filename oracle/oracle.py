"""Plain fp64 CPU oracle of the tensor-parallel sharded-linear path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, links or runs
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` do.  It shares no code with the CUDA library.

Every function is the plain definition from the pages, in float64, with numpy
``matmul`` as the only library step.  No blocking, fusion or reordering beyond
what each definition states.  bf16 inputs are read as their exact values.

Sources (pages by title, section):

* nanotron rules, "Tensor-Parallel Component Patterns" -- "MLP Module":
  c_fc is a column-parallel linear whose per-rank output has
  ``intermediate_size // tp`` columns, then ``F.gelu``, then the row-parallel
  c_proj.  "Attention Module": the row linear takes the full dimensions.
* DeepSpeed "Class SubParamLinearLayer" (deepspeed/module_inject/layers.py):
  the ``shape`` spec ``(3, -1)`` / ``((q, k, v), -1)`` with ``partition_dim=0``
  names sub-parameters that are each partitioned separately; the bias is
  partitioned like the weight's output dim and must match its size;
  ``forward`` is ``matmul(input, weight^T) + bias``.
* google-research ``two_d_parallel_xmap.py``: ``allgather_layernorm`` (RMSNorm
  with epsilon 1e-6 inside the rsqrt, optional ``scale += 1.0`` centring);
  ``unembed_manual`` (fp32 logits ``'bte,ve->btv'``); the ``o_wo`` section of
  ``transformer_layer_weight_stationary`` (per-shard partial products summed
  over the sharded contraction axis) and its ``residual`` section.
* Tenstorrent ``lm_head_1d.py``: module docstring (vocab-sharded logits; the
  argmax over devices is left to the caller) and ``LMHead1D.from_model_args``
  (per-device vocab size, split sizes, global column of a chunk).

Readings taken where the pages are silent are listed beside each function.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

try:  # the library erf; math.erf element by element if scipy is absent
    from scipy.special import erf as _erf
except ImportError:  # pragma: no cover
    _erf = np.vectorize(math.erf, otypes=[np.float64])

MAX_TP = 64
MAX_SUB = 8


class OracleError(ValueError):
    """Argument rejected by a validation rule; ``kind`` mirrors the C status names."""

    def __init__(self, kind: str, msg: str):
        super().__init__(f"{kind}: {msg}")
        self.kind = kind


# --------------------------------------------------------------------------
# a1. Sub-parameter partition (SubParamLinearLayer, shape spec and bias rule)
# --------------------------------------------------------------------------

@dataclass
class Partition:
    tp: int
    sub_sizes: List[int]
    width: List[List[int]]        # [r][j]
    src_off: List[List[int]]      # [r][j] row of the fused weight / index of the fused bias
    dst_off: List[List[int]]      # [r][j] column inside rank r's shard
    shard_width: List[int]        # [r]
    shard_base: List[int]         # [r] = sum of shard_width of lower ranks

    @property
    def logical_out(self) -> int:
        return sum(self.sub_sizes)


def partition_subparams(sub_sizes: Sequence[int], tp: int, align: int = 1) -> Partition:
    """Split each sub-parameter of a fused weight separately over ``tp`` ranks.

    SubParamLinearLayer: every logical sub-parameter (q, k, v of a fused QKV,
    possibly of unequal GQA sizes) is partitioned on its own along the output
    dim, and rank r's shard holds its piece of each sub-parameter in the given
    order.

    Reading (the page does not print the width rule): sub-parameter j is cut
    into ``S_j / align`` units of ``align`` rows (align = head_dim keeps heads
    whole); rank r gets ``units // tp`` units plus one more if
    ``r < units % tp`` (remainder to the lowest ranks).  A size not divisible
    by ``align``, or a rank left with no rows of some sub-parameter, is
    rejected (the LM-head page's ``0 < logical width`` rule).
    """
    n_sub = len(sub_sizes)
    if tp < 1 or tp > MAX_TP:
        raise OracleError("SHAPE", f"tp_size {tp} outside [1, {MAX_TP}]")
    if n_sub < 1 or n_sub > MAX_SUB:
        raise OracleError("SHAPE", f"{n_sub} sub-parameters outside [1, {MAX_SUB}]")
    if align < 1:
        raise OracleError("SHAPE", f"align {align} < 1")
    for s in sub_sizes:
        if s < 1:
            raise OracleError("SHAPE", f"sub-parameter size {s} < 1")
        if s % align != 0:
            raise OracleError("INDIVISIBLE", f"sub-parameter size {s} not a multiple of {align}")

    width = [[0] * n_sub for _ in range(tp)]
    for j, s in enumerate(sub_sizes):
        units = s // align
        for r in range(tp):
            u = units // tp + (1 if r < units % tp else 0)
            if u == 0:
                raise OracleError("INDIVISIBLE", f"rank {r} gets no rows of sub-parameter {j}")
            width[r][j] = u * align

    src_off = [[0] * n_sub for _ in range(tp)]
    dst_off = [[0] * n_sub for _ in range(tp)]
    for r in range(tp):
        for j in range(n_sub):
            src_off[r][j] = sum(sub_sizes[:j]) + sum(width[q][j] for q in range(r))
            dst_off[r][j] = sum(width[r][:j])
    shard_width = [sum(width[r]) for r in range(tp)]
    shard_base = [sum(shard_width[:r]) for r in range(tp)]
    return Partition(tp, list(sub_sizes), width, src_off, dst_off, shard_width, shard_base)


def check_bias_size(part: Partition, bias_numel: int) -> None:
    """SubParamLinearLayer: the bias must have exactly the output-shape size."""
    if bias_numel != part.logical_out:
        raise OracleError("SHAPE", f"bias size {bias_numel} != output size {part.logical_out}")


# --------------------------------------------------------------------------
# a4. GELU (nanotron MLP Module: F.gelu; tanh form for the tiny workload)
# --------------------------------------------------------------------------

def gelu_erf(y: np.ndarray) -> np.ndarray:
    """Exact GELU, y * Phi(y) = 0.5 y (1 + erf(y / sqrt 2)) (Hendrycks & Gimpel)."""
    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * (1.0 + _erf(y / math.sqrt(2.0)))


def gelu_tanh(y: np.ndarray) -> np.ndarray:
    """tanh approximation 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))."""
    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (y + 0.044715 * y ** 3)))


def activation(y: np.ndarray, act: str) -> np.ndarray:
    if act in (None, "none"):
        return np.asarray(y, dtype=np.float64)
    if act == "gelu_erf":
        return gelu_erf(y)
    if act == "gelu_tanh":
        return gelu_tanh(y)
    raise OracleError("UNSUPPORTED", f"activation {act}")


# --------------------------------------------------------------------------
# a3. Column-parallel linear (SubParamLinearLayer.forward; nanotron c_fc)
# --------------------------------------------------------------------------

def column_linear(x: np.ndarray, w: np.ndarray, bias: Optional[np.ndarray], part: Partition,
                  act: str = "none") -> List[np.ndarray]:
    """Per-rank shard outputs ``Y_r = act(X W_r^T + b_r)``.

    ``x`` is ``[M, K]``, ``w`` the unsharded fused weight ``[logical_out, K]``
    in nn.Linear layout, ``bias`` ``[logical_out]`` or None.  ``W_r`` stacks,
    for j in order, rows ``src_off[r][j] .. + width[r][j]`` of ``w``; its piece
    of the output lands at columns ``dst_off[r][j] ..`` of rank r's shard.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    if w.shape[0] != part.logical_out or w.shape[1] != x.shape[1]:
        raise OracleError("SHAPE", f"weight {w.shape} vs out {part.logical_out}, K {x.shape[1]}")
    if bias is not None:
        check_bias_size(part, int(np.asarray(bias).size))
        bias = np.asarray(bias, dtype=np.float64)
    M = x.shape[0]
    out = []
    for r in range(part.tp):
        y = np.zeros((M, part.shard_width[r]), dtype=np.float64)
        for j in range(len(part.sub_sizes)):
            s, d, n = part.src_off[r][j], part.dst_off[r][j], part.width[r][j]
            piece = x @ w[s:s + n].T
            if bias is not None:
                piece = piece + bias[s:s + n]
            y[:, d:d + n] = piece
        out.append(activation(y, act))
    return out


# --------------------------------------------------------------------------
# a5. Row-parallel linear with the partial-sum reduction (o_wo; c_proj)
# --------------------------------------------------------------------------

def row_partials(h: Sequence[np.ndarray], w2: Sequence[np.ndarray]) -> List[np.ndarray]:
    """Per-rank partial products ``P_r = H_r W2_r^T`` ({YZ unreduced} in o_wo).

    ``h[r]`` is ``[M, k_r]`` (rank r's slice of the contraction dim),
    ``w2[r]`` is ``[N, k_r]``: columns ``koff_r .. koff_r + k_r`` of the
    unsharded ``[N, K]`` weight.
    """
    if len(h) != len(w2):
        raise OracleError("SHAPE", "h and w2 have different rank counts")
    parts = []
    for hr, wr in zip(h, w2):
        hr = np.asarray(hr, dtype=np.float64)
        wr = np.asarray(wr, dtype=np.float64)
        if hr.shape[1] != wr.shape[1]:
            raise OracleError("SHAPE", f"rank slice widths {hr.shape[1]} != {wr.shape[1]}")
        parts.append(hr @ wr.T)
    return parts


def row_linear_reduce(h: Sequence[np.ndarray], w2: Sequence[np.ndarray],
                      bias: Optional[np.ndarray] = None,
                      residual: Optional[np.ndarray] = None) -> np.ndarray:
    """``Y = sum_r P_r (+ b) (+ R)``, the sum taken in rank order.

    Readings: the reduction is the full sum over ranks (one GPU, no
    reduce-scatter); a bias is added once after the sum; the residual is the
    ``z = y_out + x`` of the residual section.
    """
    parts = row_partials(h, w2)
    y = np.zeros_like(parts[0])
    for p in parts:
        y = y + p
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    if residual is not None:
        y = y + np.asarray(residual, dtype=np.float64)
    return y


def row_weight_slices(w2_full: np.ndarray, k_w: Sequence[int]) -> List[np.ndarray]:
    """Rank r's ``[N, k_r]`` column slice of an unsharded ``[N, K]`` weight."""
    out, off = [], 0
    for k in k_w:
        out.append(np.asarray(w2_full)[:, off:off + k])
        off += k
    return out


# --------------------------------------------------------------------------
# a2. RMSNorm (allgather_layernorm; weight-gathered layernorm section)
# --------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, scale: Optional[np.ndarray] = None, centered: bool = False,
            eps: float = 1e-6) -> np.ndarray:
    """``y = x / sqrt(mean(x^2) + eps) * g``, g = 1 + s (centred), s, or 1.

    Reading: the page rounds the normalised value to bf16 before scaling and
    again after; the oracle keeps float64 throughout (no intermediate rounding).
    """
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if scale is not None:
        g = np.asarray(scale, dtype=np.float64)
        if centered:
            g = g + 1.0
        y = y * g
    return y


# --------------------------------------------------------------------------
# a6. Vocab-sharded, chunked LM head with per-shard and global argmax
# --------------------------------------------------------------------------

@dataclass
class VocabLayout:
    vocab: int
    tp: int
    shard: int                 # ids per shard (last shard may hold fewer real ids)
    split_sizes: List[int]     # columns of each chunk of a shard

    def global_id(self, r: int, chunk: int, j: int) -> int:
        """Global column of column j of chunk ``chunk`` on shard r."""
        return r * self.shard + sum(self.split_sizes[:chunk]) + j


def vocab_layout(vocab: int, tp: int, n_chunks: int) -> VocabLayout:
    """Per-shard vocab size and chunk split sizes (LMHead1D.from_model_args).

    Reading: B200 needs no tile padding, so the page's tile is 1 and
    ``shard = ceil(V / tp)``.  The page derives the number of splits from a
    column cap; here the caller gives the number of chunks, the cap is
    ``ceil(shard / n_chunks)``, and the page's formula must give back exactly
    n_chunks splits with a positive last width.
    """
    if vocab < 1 or tp < 1 or tp > MAX_TP or n_chunks < 1:
        raise OracleError("SHAPE", f"vocab {vocab}, tp {tp}, n_chunks {n_chunks}")
    shard = -(-vocab // tp)
    cap = -(-shard // n_chunks)
    num_splits = -(-shard // cap)
    split = [min(shard, cap)] * (num_splits - 1)
    split.append(shard - sum(split))
    if num_splits != n_chunks or split[-1] <= 0:
        raise OracleError("SHAPE", f"shard {shard} does not split into {n_chunks} chunks")
    return VocabLayout(vocab, tp, shard, split)


@dataclass
class LMHeadResult:
    logits: np.ndarray          # [B, V] float64
    shard_max: np.ndarray       # [tp, B] (-inf for a shard with no real ids)
    shard_idx: np.ndarray       # [tp, B] global ids (-1 for an empty shard)
    ids: np.ndarray             # [B]
    gap: np.ndarray             # [B] top-1 minus top-2 logit over the whole vocab
    shard_gap: np.ndarray       # [tp, B] same, within each shard (inf if < 2 ids)


def lmhead_logits(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """``logits[b, v] = x[b] . W[v]`` (unembed_manual: 'bte,ve->btv')."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def _top2(vals: np.ndarray):
    """Index of the largest value (lowest index on ties) and its gap to the next."""
    i = int(np.argmax(vals))
    if vals.size < 2:
        return i, math.inf
    rest = np.delete(vals, i)
    return i, float(vals[i] - rest.max())


def lmhead_argmax(x: np.ndarray, w: np.ndarray, tp: int, n_chunks: int,
                  logits: Optional[np.ndarray] = None) -> LMHeadResult:
    """Per-shard argmax, then the global argmax over shards.

    Readings: ties go to the lowest global id (within a shard and across
    shards); ids at or beyond V are never reported; a shard that holds no real
    id reports max -inf and id -1.
    """
    B, K = np.asarray(x).shape
    V = np.asarray(w).shape[0] if logits is None else logits.shape[1]
    lay = vocab_layout(V, tp, n_chunks)
    if logits is None:
        logits = lmhead_logits(x, w)
    shard_max = np.full((tp, B), -np.inf)
    shard_idx = np.full((tp, B), -1, dtype=np.int64)
    shard_gap = np.full((tp, B), np.inf)
    for r in range(tp):
        lo, hi = r * lay.shard, min((r + 1) * lay.shard, V)
        if lo >= hi:
            continue
        for b in range(B):
            i, g = _top2(logits[b, lo:hi])
            shard_max[r, b] = logits[b, lo + i]
            shard_idx[r, b] = lo + i
            shard_gap[r, b] = g
    ids = np.zeros(B, dtype=np.int64)
    gap = np.zeros(B)
    for b in range(B):
        best = -1
        for r in range(tp):
            if shard_idx[r, b] < 0:
                continue
            if best < 0 or shard_max[r, b] > shard_max[best, b]:
                best = r
        ids[b] = shard_idx[best, b]
        _, gap[b] = _top2(logits[b])
    return LMHeadResult(logits, shard_max, shard_idx, ids, gap, shard_gap)


# --------------------------------------------------------------------------
# a7. MLP block and layer stack (nanotron MLP Module; o_wo residual section)
# --------------------------------------------------------------------------

def tp_mlp(x: np.ndarray, w1: np.ndarray, w2_full: np.ndarray, tp: int, act: str,
           scale: Optional[np.ndarray] = None, centered: bool = False, norm: bool = False,
           residual: bool = False, eps: float = 1e-6) -> np.ndarray:
    """One block: ``[x +] c_proj(act(c_fc(norm(x))))`` with tp shards of each linear."""
    x = np.asarray(x, dtype=np.float64)
    xn = rmsnorm(x, scale, centered, eps) if norm else x
    part = partition_subparams([w1.shape[0]], tp, 1)
    h = column_linear(xn, w1, None, part, act)
    w2 = row_weight_slices(w2_full, part.shard_width)
    return row_linear_reduce(h, w2, None, x if residual else None)


def tp_stack(x: np.ndarray, layers: Sequence[tuple], tp: int, act: str, eps: float = 1e-6,
             centered: bool = False) -> np.ndarray:
    """``x <- x + MLP(RMSNorm(x))`` per layer; ``layers`` holds (w1, w2, scale|None).

    The oracle keeps x in float64 between layers.
    """
    x = np.asarray(x, dtype=np.float64)
    for (w1, w2, s) in layers:
        x = tp_mlp(x, w1, w2, tp, act, scale=s, centered=centered, norm=True, residual=True,
                   eps=eps)
    return x


def rel_frobenius(got: np.ndarray, ref: np.ndarray) -> float:
    """``||G - O||_F / ||O||_F`` in float64."""
    g = np.asarray(got, dtype=np.float64)
    o = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm((g - o).ravel()) / np.linalg.norm(o.ravel()))


# --------------------------------------------------------------------------
# Next rows: sequence-parallel layouts, SwiGLU, vocab-sharded embedding
# --------------------------------------------------------------------------

def seq_scatter(y: np.ndarray, batch: int, seq: int, tp: int) -> np.ndarray:
    """Rank-major sequence slices ``[tp][batch][seq/tp][N]`` of ``y [batch*seq, N]``.

    nanotron "MLP Module": the row-parallel c_proj hands each rank the output
    rows ``[batch, seq // tp, hidden]`` -- after the sum over ranks, rank r
    keeps tokens ``r*seq/tp .. (r+1)*seq/tp`` of every sequence (a
    reduce-scatter along the sequence).
    """
    y = np.asarray(y)
    if seq % tp != 0:
        raise OracleError("INDIVISIBLE", f"seq {seq} not divisible by tp {tp}")
    n = y.shape[1]
    return y.reshape(batch, tp, seq // tp, n).transpose(1, 0, 2, 3).copy()


def seq_gather(x_sp: np.ndarray, batch: int, seq: int, tp: int) -> np.ndarray:
    """Inverse of :func:`seq_scatter`: ``[batch*seq, N]`` from rank-major slices
    (the all-gather along the sequence ahead of a column-parallel linear)."""
    x_sp = np.asarray(x_sp)
    n = x_sp.shape[-1]
    return x_sp.reshape(tp, batch, seq // tp, n).transpose(1, 0, 2, 3).reshape(batch * seq, n)


def row_linear_reduce_scatter(h, w2, batch: int, seq: int, bias=None,
                              residual_sp=None) -> np.ndarray:
    """Row-parallel linear whose summed output is scattered along the sequence.

    Returns ``[tp][batch][seq/tp][N]``; a residual is given in the same layout.
    """
    tp = len(h)
    y = row_linear_reduce(h, w2, bias, None)
    out = seq_scatter(y, batch, seq, tp)
    if residual_sp is not None:
        out = out + np.asarray(residual_sp, dtype=np.float64)
    return out


def column_linear_allgather(x_sp, batch: int, seq: int, w, bias, part: Partition,
                            act: str = "none") -> List[np.ndarray]:
    """Column-parallel linear of sequence-sharded activations (gather, then a3)."""
    return column_linear(seq_gather(x_sp, batch, seq, part.tp), w, bias, part, act)


def silu(a: np.ndarray) -> np.ndarray:
    """Swish with beta = 1: a * sigmoid(a) (the gate of SwiGLU)."""
    a = np.asarray(a, dtype=np.float64)
    return a / (1.0 + np.exp(-a))


def swiglu_column_linear(x: np.ndarray, w: np.ndarray, F: int, tp: int) -> List[np.ndarray]:
    """Column-parallel fused SwiGLU projection (google-research "SwiGLU" section).

    ``w`` is the fused ``[wi0; wi1]`` weight ``[2F, K]``; it is partitioned as
    two equal sub-parameters, rank r holding its slice of each, and returns
    ``h_r = silu(X wi0_r^T) * (X wi1_r^T)``, ``[M, F_r]`` per rank.
    Reading: "swish2" is taken as swish with beta = 1 (SiLU).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    if w.shape[0] != 2 * F:
        raise OracleError("SHAPE", f"fused weight has {w.shape[0]} rows, expected {2 * F}")
    part = partition_subparams([F, F], tp, 1)
    out = []
    for r in range(tp):
        s0, n = part.src_off[r][0], part.width[r][0]
        s1 = part.src_off[r][1]
        a = x @ w[s0:s0 + n].T
        b = x @ w[s1:s1 + n].T
        out.append(silu(a) * b)
    return out


def embedding_lookup(ids: np.ndarray, table: np.ndarray, tp: int) -> np.ndarray:
    """Vocab-sharded embedding (google-research ``embed_manual``, 'embed' scope).

    Each rank r holds rows ``r*shard .. (r+1)*shard`` of the table; it looks up
    ``one_x = x - vocab_start`` and keeps the row only where
    ``0 <= one_x < shard_rows``; the sum over ranks is the embedding.  Ids
    outside ``[0, V)`` embed to zeros.
    """
    ids = np.asarray(ids).reshape(-1)
    table = np.asarray(table, dtype=np.float64)
    V, H = table.shape
    shard = -(-V // tp)
    out = np.zeros((ids.size, H))
    for r in range(tp):
        start = r * shard
        rows = max(0, min(shard, V - start))
        for i, tok in enumerate(ids):
            local = int(tok) - start
            if 0 <= local < rows:
                out[i] += table[start + local]
    return out
