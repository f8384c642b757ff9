"""Element-wise error bounds of the GPU path against the fp64 oracle.

Next to the relative Frobenius tolerance (which a handful of wrong elements in
a large output can stay under), every compared element must satisfy a bound
derived from the path's arithmetic:

    |G - O| <= MARGIN * (u |O| + own + LAMBDA * sqrt(carried))

* ``u |O|``: the output's own rounding on store (round to nearest even; unit
  roundoff ``U_BF16 = 2^-8`` for bf16's 8-bit significand, ``U_FP32 = 2^-24``).
* ``own``: the last step's own arithmetic, worst case.  An fp32 dot product
  of length K accumulated by the tensor cores as ceil(K/16) sequential fp32
  additions of 16-term partial sums (K additions in the SIMT kernel) errs by
  at most ``acc(K) * sum_k |a_k b_k|`` with ``acc(K) = (steps + 16) U_FP32``
  (the 16 covers the partial-sum tree, the bias add and the epilogue's own
  roundings).  GELU's derivative is at most 1.13 in magnitude (1.1289 at
  y = 2.42 for the erf form; the tanh form stays below it) and its evaluation
  in the epilogue (hardware exp and divide) adds at most ``ACT_APPROX |y|``.
  RMSNorm in fp32 over H values errs by at most ``(H/2 + 8) U_FP32`` relative.
* ``carried``: errors already in a step's inputs (the bf16 rounding of an
  intermediate such as RMSNorm's output or the hidden h, or an earlier
  layer's error), carried through the following contractions.  Bounding those
  sums in absolute value makes the bound of a multi-step path vacuous (several
  times |O| after two contractions), so they follow the probabilistic model of
  rounding errors (Higham & Mary, "A new approach to probabilistic rounding
  error analysis", SIAM J. Sci. Comput. 2019): errors of different elements are
  independent with mean zero and bounded by their worst-case bounds e_k, so a
  combination sum_k c_k d_k is sub-Gaussian with variance proxy
  sum_k c_k^2 e_k^2.  Proxies add through every later step, and Hoeffding's
  inequality bounds the carried error by LAMBDA * sqrt(proxy) except with
  probability 2 exp(-LAMBDA^2 / 2) (2.5e-14 per element for LAMBDA = 8).

The scale terms ``sum |a||b|`` and ``sum c^2 e^2`` are the oracle's own
contractions applied to absolute values and squares, so shards, pieces and
partitions are handled exactly as the oracle handles them.  Second-order terms
are covered by a 5 % margin.  An element over its bound fails with its index
and values.
"""
import math
from typing import Optional, Sequence

import numpy as np

import oracle as O

U_BF16 = 2.0 ** -8
U_FP32 = 2.0 ** -24
ACT_SLOPE = 1.13
ACT_APPROX = 4e-6
MARGIN = 1.05
LAMBDA = 8.0


def acc(K: int, simt: bool = False) -> float:
    """fp32 accumulation error coefficient of a length-K dot product."""
    steps = K if simt else math.ceil(K / 16)
    return (steps + 16) * U_FP32


def norm_err(H: int) -> float:
    """Relative error of the fp32 RMSNorm factor over H values."""
    return (H / 2 + 8) * U_FP32


def bound(ref, own=0.0, carried=None, u_out: float = U_BF16):
    o = np.abs(np.asarray(ref, dtype=np.float64))
    b = u_out * o + own
    if carried is not None:
        b = b + LAMBDA * np.sqrt(carried)
    return MARGIN * b


def check(got, ref, own=0.0, carried=None, u_out: float = U_BF16, what: str = "") -> float:
    """Asserts |G - O| <= bound(O, own, carried, u_out) element by element;
    returns the largest ratio of error to bound."""
    g = np.asarray(got, dtype=np.float64)
    o = np.asarray(ref, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    b = bound(o, own, carried, u_out) + 1e-300
    ratio = np.abs(g - o) / b
    if ratio.size == 0:
        return 0.0
    i = int(np.argmax(ratio))
    worst = float(ratio.flat[i])
    assert worst <= 1.0, (f"{what}: element {np.unravel_index(i, o.shape)} got {g.flat[i]!r} "
                          f"oracle {o.flat[i]!r} bound {b.flat[i]!r}")
    return worst


def _abs(a):
    return None if a is None else np.abs(np.asarray(a, dtype=np.float64))


def _sq(a):
    return None if a is None else np.square(np.asarray(a, dtype=np.float64))


def column(x, w, bias, part, act: str = "none", simt: bool = False, x_proxy=None):
    """Column-parallel linear: (reference shards, own, carried) per rank.
    ``x_proxy``: variance proxy of the error already in x."""
    K = x.shape[1]
    ref = O.column_linear(x, w, bias, part, act)
    z = O.column_linear(x, w, bias, part, "none") if act != "none" else ref
    s = O.column_linear(_abs(x), _abs(w), _abs(bias), part, "none")
    p = None if x_proxy is None else O.column_linear(x_proxy, _sq(w), None, part, "none")
    own, car = [], []
    for r in range(part.tp):
        e = acc(K, simt) * s[r]
        c = None if p is None else p[r]
        if act != "none":
            e = ACT_SLOPE * e + ACT_APPROX * np.abs(z[r])
            c = None if c is None else ACT_SLOPE ** 2 * c
        own.append(e)
        car.append(c)
    return ref, own, car


def row(hs: Sequence[np.ndarray], ws: Sequence[np.ndarray], bias=None, res=None,
        simt: bool = False, h_proxy: Optional[Sequence[np.ndarray]] = None):
    """Row-parallel linear with its partial-sum reduction (+ bias, + residual):
    (reference, own, carried).  ``h_proxy``: variance proxies of the errors
    already in each rank's input block."""
    ref = O.row_linear_reduce(hs, ws, bias, res)
    s = O.row_linear_reduce([_abs(h) for h in hs], [_abs(w) for w in ws], _abs(bias), _abs(res))
    K = sum(h.shape[1] for h in hs)
    car = None if h_proxy is None else O.row_linear_reduce(list(h_proxy), [_sq(w) for w in ws])
    return ref, acc(K, simt) * s, car


def partials(hs, ws, simt: bool = False):
    """Each rank's fp32 partial alone: (reference partials, own per rank)."""
    ref = O.row_partials(hs, ws)
    s = O.row_partials([_abs(h) for h in hs], [_abs(w) for w in ws])
    return ref, [acc(h.shape[1], simt) * si for h, si in zip(hs, s)]


def rmsnorm(x, scale=None, centered=False, eps=1e-6):
    """(reference, own) of RMSNorm computed in fp32."""
    ref = O.rmsnorm(x, scale, centered, eps)
    return ref, norm_err(x.shape[1]) * np.abs(ref)


def logits(x, w):
    """Own error of fp32 logits x . W^T from bf16 inputs."""
    return acc(x.shape[1]) * (_abs(x) @ _abs(w).T)


def stored(ref, own, carried, u: float):
    """Variance proxy of an intermediate after it is stored (rounded by u):
    its own errors and its rounding become errors carried by the next step."""
    p = np.square(own + u * np.abs(ref))
    return p if carried is None else p + carried


def mlp(x, w1, w2_full, tp, act, scale=None, centered=False, norm=False, residual=False,
        eps=1e-6, x_proxy=None, bf16=True, align=1):
    """``[x +] c_proj(act(c_fc([RMSNorm] x)))``: (reference y, own, carried).

    bf16: RMSNorm's output and h are stored in bf16 between the steps (fp32 for
    the fp32 path); y is rounded once on store.  ``x_proxy``: variance proxy of
    an error already in x (the stack's earlier layers)."""
    x = np.asarray(x, dtype=np.float64)
    H = x.shape[1]
    u = U_BF16 if bf16 else U_FP32
    simt = not bf16
    part = O.partition_subparams([w1.shape[0]], tp, align)
    if norm:
        xn, own_n = rmsnorm(x, scale, centered, eps)
        car_n = None
        if x_proxy is not None:
            # first order in dx: d xn = (g / rms) dx - xn (x . dx) / (H (ms + eps))
            ms = np.mean(x * x, axis=1, keepdims=True)
            g = np.ones(H) if scale is None else (1.0 + scale if centered else scale)
            car_n = (np.square(g) / (ms + eps)) * x_proxy + np.square(xn) * (
                np.sum(np.square(x) * x_proxy, axis=1, keepdims=True) / np.square(H * (ms + eps)))
        xn_proxy = stored(xn, own_n, car_n, u)
    else:
        xn, xn_proxy = x, x_proxy
    h_ref, own_h, car_h = column(xn, w1, None, part, act, simt=simt, x_proxy=xn_proxy)
    h_proxy = [stored(h, o, c, u) for h, o, c in zip(h_ref, own_h, car_h)]
    w2 = O.row_weight_slices(w2_full, part.shard_width)
    y, own_y, car_y = row(h_ref, w2, None, x if residual else None, simt=simt, h_proxy=h_proxy)
    if residual and x_proxy is not None:
        car_y = car_y + x_proxy
    return y, own_y, car_y


def stack(x, layers, tp, act, eps=1e-6):
    """Residual stack ``x <- x + MLP(RMSNorm(x))``, x stored in bf16 after every
    layer: (reference after the last layer, own, carried)."""
    x = np.asarray(x, dtype=np.float64)
    proxy = None
    for i, (w1, w2) in enumerate(layers):
        y, own, car = mlp(x, w1, w2, tp, act, norm=True, residual=True, eps=eps, x_proxy=proxy)
        if i + 1 < len(layers):
            proxy = stored(y, own, car, U_BF16)
        x = y
    return x, own, car


def swiglu(x, w, F, tp):
    """Fused SwiGLU column linear h_r = silu(a) * b, a = X wi0_r^T, b = X wi1_r^T:
    (reference shards, own) per rank.  d(silu(a) b) = silu'(a) b da + silu(a) db
    with |silu'| <= 1.1 (1.0998 at a = 2.40)."""
    K = x.shape[1]
    ref = O.swiglu_column_linear(x, w, F, tp)
    part = O.partition_subparams([F, F], tp, 1)
    xa, wa = _abs(x), _abs(w)
    own = []
    for r in range(tp):
        s0, n, s1 = part.src_off[r][0], part.width[r][0], part.src_off[r][1]
        a = x @ w[s0:s0 + n].T
        b = x @ w[s1:s1 + n].T
        ea = acc(K) * (xa @ wa[s0:s0 + n].T)
        eb = acc(K) * (xa @ wa[s1:s1 + n].T)
        own.append(1.1 * ea * np.abs(b) + np.abs(O.silu(a)) * eb + ACT_APPROX * np.abs(ref[r]))
    return ref, own


def scatter_reduce(hs, ws, bias=None, res=None):
    """The row-parallel linear over GPUs: every rank's partial is stored in
    bf16 (a slot of its owner's receive buffer), then the slots, the bias and
    the residual are summed in fp32 and rounded once: (reference, own, carried)."""
    parts = O.row_partials(hs, ws)
    s = O.row_partials([_abs(h) for h in hs], [_abs(w) for w in ws])
    tp = len(hs)
    ref = sum(parts)
    terms = sum(np.abs(p) for p in parts)
    if bias is not None:
        ref = ref + bias
        terms = terms + np.abs(bias)
    if res is not None:
        ref = ref + res
        terms = terms + np.abs(res)
    own = (tp + 2) * U_FP32 * terms
    carried = sum(np.square(acc(h.shape[1]) * si + U_BF16 * np.abs(p))
                  for h, si, p in zip(hs, s, parts))
    return ref, own, carried


def slot_sum(slots, res=None):
    """Sum of bf16 slots (+ residual) in fp32, rounded once: (reference, own)."""
    slots = [np.asarray(sl, dtype=np.float64) for sl in slots]
    ref = sum(slots)
    terms = sum(np.abs(sl) for sl in slots)
    if res is not None:
        ref = ref + res
        terms = terms + np.abs(res)
    return ref, (len(slots) + 2) * U_FP32 * terms


def rank_mlp(x, w1, w2_full, tp, act, scale=None, centered=False, eps=1e-6, x_proxy=None):
    """The MLP block over GPUs (RMSNorm -> c_fc + act -> c_proj, each rank's
    c_proj partial stored in bf16 in its owner's slot, the slots and the
    residual summed in fp32 and rounded once): (reference y, own, carried)."""
    x = np.asarray(x, dtype=np.float64)
    H = x.shape[1]
    part = O.partition_subparams([w1.shape[0]], tp, 1)
    xn, own_n = rmsnorm(x, scale, centered, eps)
    car_n = None
    if x_proxy is not None:
        ms = np.mean(x * x, axis=1, keepdims=True)
        g = np.ones(H) if scale is None else (1.0 + scale if centered else scale)
        car_n = (np.square(g) / (ms + eps)) * x_proxy + np.square(xn) * (
            np.sum(np.square(x) * x_proxy, axis=1, keepdims=True) / np.square(H * (ms + eps)))
    h_ref, own_h, car_h = column(xn, w1, None, part, act, x_proxy=stored(xn, own_n, car_n, U_BF16))
    h_proxy = [stored(h, o, c, U_BF16) for h, o, c in zip(h_ref, own_h, car_h)]
    w2 = O.row_weight_slices(w2_full, part.shard_width)
    parts = O.row_partials(h_ref, w2)
    s = O.row_partials([_abs(h) for h in h_ref], [_abs(w) for w in w2])
    car_p = [O.row_partials([hp], [_sq(w)])[0] for hp, w in zip(h_proxy, w2)]
    y = sum(parts) + x
    own = (tp + 2) * U_FP32 * (sum(np.abs(p) for p in parts) + np.abs(x))
    car = sum(stored(p, acc(h.shape[1]) * si, cp, U_BF16)
              for p, h, si, cp in zip(parts, h_ref, s, car_p))
    if x_proxy is not None:
        car = car + x_proxy
    return y, own, car
