"""The five synthetic workloads of the sharded-linear path, by shape.

Each workload is named by what it is, with its sizes.  Shapes follow the pages:
hidden states arrive as ``[batch, seq, hidden]`` and are flattened to
``M = batch * seq`` rows; weights use the ``nn.Linear`` layout ``[out, in]``.
Value distributions: activations ~N(0,1), weights ~N(0, sigma), the RMSNorm
scale ~N(0, 0.1) applied with the centred (``1 + s``) convention, bias
~N(0, 0.02).  All tensors come from :mod:`workloads.gen` with seed 0.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch

from . import gen


@dataclass(frozen=True)
class MLPWorkload:
    """RMSNorm (optional) -> column-parallel c_fc + GELU -> row-parallel c_proj."""
    name: str
    batch: int
    seq: int
    hidden: int
    inter: int
    tp: int
    act: str                      # "gelu_erf" | "gelu_tanh"
    w_sigma: float
    dtype: torch.dtype
    norm: bool                    # RMSNorm ahead of c_fc
    norm_scale: bool              # a learned scale (centred) is applied
    residual: bool                # x + MLP(x)
    layers: int = 1

    @property
    def M(self) -> int:
        return self.batch * self.seq

    def flops(self) -> float:
        return self.layers * 2 * (2.0 * self.M * self.hidden * self.inter)


@dataclass(frozen=True)
class QKVWorkload:
    """Column-parallel fused QKV projection with per-sub-parameter partitioning."""
    name: str
    batch: int
    seq: int
    hidden: int
    sub_sizes: Tuple[int, ...]
    align: int
    tp: int
    w_sigma: float
    bias_sigma: float

    @property
    def M(self) -> int:
        return self.batch * self.seq

    @property
    def out(self) -> int:
        return sum(self.sub_sizes)

    def flops(self) -> float:
        return 2.0 * self.M * self.hidden * self.out


@dataclass(frozen=True)
class LMHeadWorkload:
    """Decode LM head over a vocab split into tp shards of n_chunks chunks each."""
    name: str
    batch: int
    hidden: int
    vocab: int
    tp: int
    n_chunks: int
    w_sigma: float

    def weight_bytes(self) -> int:
        return self.vocab * self.hidden * 2

    def algorithmic_bytes(self, with_logits: bool = False) -> int:
        # W and x are read once; ids, per-shard max and per-shard ids written.
        b = self.weight_bytes() + self.batch * self.hidden * 2
        b += self.batch * 4 + 2 * self.tp * self.batch * 4
        if with_logits:
            b += self.batch * self.vocab * 4
        return b

    def flops(self) -> float:
        return 2.0 * self.batch * self.hidden * self.vocab


TINY_MLP = MLPWorkload("tiny-tp-mlp x[2,16,256] fp32 256->1024->256 tp4 gelu-tanh",
                       batch=2, seq=16, hidden=256, inter=1024, tp=4, act="gelu_tanh",
                       w_sigma=0.02, dtype=torch.float32, norm=False, norm_scale=False,
                       residual=False)

GQA_QKV = QKVWorkload("gqa-fused-qkv x[4,1024,4096] bf16 q4096+k1024+v1024 tp8",
                      batch=4, seq=1024, hidden=4096, sub_sizes=(4096, 1024, 1024), align=128,
                      tp=8, w_sigma=0.02, bias_sigma=0.02)

TP_MLP = MLPWorkload("rmsnorm-tp-mlp x[8,1024,4096] bf16 4096->14336->4096 tp8 gelu-erf",
                     batch=8, seq=1024, hidden=4096, inter=14336, tp=8, act="gelu_erf",
                     w_sigma=0.02, dtype=torch.bfloat16, norm=True, norm_scale=True,
                     residual=False)

LM_HEAD = LMHeadWorkload("decode-lmhead x[32,4096] W[128256,4096] bf16 tp8x4chunks",
                         batch=32, hidden=4096, vocab=128256, tp=8, n_chunks=4, w_sigma=0.02)

STACK4 = MLPWorkload("4-layer-tp-stack x[4,4096,8192] bf16 8192->28672->8192 tp8 gelu-erf",
                     batch=4, seq=4096, hidden=8192, inter=28672, tp=8, act="gelu_erf",
                     w_sigma=0.01, dtype=torch.bfloat16, norm=True, norm_scale=False,
                     residual=True, layers=4)

# One layer of the stack on a quarter of its tokens: the same two GEMM shapes in
# K and N with about 1.3 GB on the device, small enough for a multi-pass
# profiler capture.
STACK_LAYER = MLPWorkload("1-layer-of-tp-stack x[1,4096,8192] bf16 8192->28672->8192 tp8 "
                          "gelu-erf", batch=1, seq=4096, hidden=8192, inter=28672, tp=8,
                          act="gelu_erf", w_sigma=0.01, dtype=torch.bfloat16, norm=True,
                          norm_scale=False, residual=True, layers=1)

ALL = (TINY_MLP, GQA_QKV, TP_MLP, LM_HEAD, STACK4)


def layer_tid(base: int, layer: int) -> int:
    return base + 16 * layer


# ---- tensor materialisation (host or device; identical bits either way) ----

def mlp_x(w: MLPWorkload, device="cpu"):
    return gen.normal((w.M, w.hidden), 1.0, tensor_id=gen.TID_X, dtype=w.dtype, device=device)


def mlp_w1(w: MLPWorkload, layer=0, device="cpu"):
    return gen.normal((w.inter, w.hidden), w.w_sigma, tensor_id=layer_tid(gen.TID_W1, layer),
                      dtype=w.dtype, device=device)


def mlp_w2(w: MLPWorkload, layer=0, device="cpu"):
    """c_proj weight in nn.Linear layout ``[hidden, inter]`` (unsharded)."""
    return gen.normal((w.hidden, w.inter), w.w_sigma, tensor_id=layer_tid(gen.TID_W2, layer),
                      dtype=w.dtype, device=device)


def mlp_scale(w: MLPWorkload, layer=0, device="cpu") -> Optional[torch.Tensor]:
    if not w.norm_scale:
        return None
    return gen.normal((w.hidden,), 0.1, tensor_id=layer_tid(gen.TID_SCALE, layer),
                      dtype=torch.float32, device=device)


def qkv_x(w: QKVWorkload, device="cpu"):
    return gen.normal((w.M, w.hidden), 1.0, tensor_id=gen.TID_X, device=device)


def qkv_w(w: QKVWorkload, device="cpu"):
    return gen.normal((w.out, w.hidden), w.w_sigma, tensor_id=gen.TID_W1, device=device)


def qkv_bias(w: QKVWorkload, device="cpu"):
    return gen.normal((w.out,), w.bias_sigma, tensor_id=gen.TID_BIAS, device=device)


def lm_x(w: LMHeadWorkload, device="cpu"):
    return gen.normal((w.batch, w.hidden), 1.0, tensor_id=gen.TID_X, device=device)


def lm_w(w: LMHeadWorkload, device="cpu"):
    return gen.normal((w.vocab, w.hidden), w.w_sigma, tensor_id=gen.TID_W1, device=device)
