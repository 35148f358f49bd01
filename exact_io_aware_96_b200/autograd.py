"""torch.autograd wrappers over libfa.so.

``flash_attn_func(q, k, v, causal)`` on [B, S, H, D] tensors and
``flash_attn_qkvpacked_func(qkv, causal)`` on a packed [B, S, 3, H, D] tensor,
the two call forms the pages use ([P1] "实战集成": qkvpacked, output
[B, S, H, D], ``loss.backward()``; [P4] §4/§5: ``flash_attn_func`` on
(batch, seq_len, num_heads, head_dim) with a causal flag). The forward saves
only q, k, v, O and the per-row logsumexp; the backward rebuilds P from the
logsumexp ([P4] §3.1; [P1] "性能引擎" recomputation). All arithmetic runs in the
library's kernels; these classes only marshal tensors.

Page legend: [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练";
[P4] the FlashAttention-2 walkthrough titled "企业官网建设流程全解析".
"""
from __future__ import annotations

import torch

from . import fa


def _kernel_ready(t: torch.Tensor) -> torch.Tensor:
    """A [B, S, H, D] view the kernels accept: last axis contiguous and every
    stride a multiple of 8 elements (copy otherwise)."""
    ok = t.stride(3) == 1 and all(s % 8 == 0 for s in t.stride()[:3]) and t.data_ptr() % 16 == 0
    return t if ok else t.contiguous()


class FlashAttentionFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal: bool, scale, deterministic: bool = False):
        q, k, v = _kernel_ready(q), _kernel_ready(k), _kernel_ready(v)
        o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale, ctx.deterministic = causal, scale, deterministic
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = fa.backward(q, k, v, o, lse, _kernel_ready(do), causal=ctx.causal, scale=ctx.scale,
                                 deterministic=ctx.deterministic)
        return dq, dk, dv, None, None, None


class FlashAttentionQKVPackedFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, qkv, causal: bool, scale):
        qkv = _kernel_ready_packed(qkv)
        q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
        o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
        ctx.save_for_backward(qkv, o, lse)
        ctx.causal, ctx.scale = causal, scale
        return o

    @staticmethod
    def backward(ctx, do):
        qkv, o, lse = ctx.saved_tensors
        q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
        dqkv = torch.empty_like(qkv)
        fa.backward(q, k, v, o, lse, _kernel_ready(do), causal=ctx.causal, scale=ctx.scale,
                    dq=dqkv[:, :, 0], dk=dqkv[:, :, 1], dv=dqkv[:, :, 2])
        return dqkv, None, None


def _kernel_ready_packed(qkv: torch.Tensor) -> torch.Tensor:
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError("qkv must be [B, S, 3, H, D]")
    ok = qkv.stride(4) == 1 and all(s % 8 == 0 for s in qkv.stride()[:4]) and qkv.data_ptr() % 16 == 0
    return qkv if ok else qkv.contiguous()


def flash_attn_func(q, k, v, causal: bool = False, softmax_scale=None, deterministic: bool = False):
    """O = softmax(scale q k^T [+ causal mask]) v on [B, S, H, D] CUDA tensors, differentiable.
    ``deterministic=True`` makes the backward's dq bit-reproducible."""
    scale = q.shape[-1] ** -0.5 if softmax_scale is None else float(softmax_scale)
    return FlashAttentionFunction.apply(q, k, v, bool(causal), scale, bool(deterministic))


def flash_attn_qkvpacked_func(qkv, causal: bool = False, softmax_scale=None):
    """Attention on a packed [B, S, 3, H, D] tensor; returns [B, S, H, D]; differentiable."""
    scale = qkv.shape[-1] ** -0.5 if softmax_scale is None else float(softmax_scale)
    return FlashAttentionQKVPackedFunction.apply(qkv, bool(causal), scale)


class PackedQKVAttention(torch.nn.Module):
    """nn.Module form of ``flash_attn_qkvpacked_func`` (attention only, no projections)."""

    def __init__(self, causal: bool = False, softmax_scale=None):
        super().__init__()
        self.causal, self.softmax_scale = causal, softmax_scale

    def forward(self, qkv):
        return flash_attn_qkvpacked_func(qkv, self.causal, self.softmax_scale)
