"""Seeded synthetic inputs and the workload table.

This module holds no attention arithmetic: it only draws random tensors of the
shapes the workloads name, so that the CUDA path and the CPU oracle can be fed
identical data. Both the tests and ``bench.py`` use it.

Workloads (shapes from the usage snippets of the pages, see the legend below):

* ``c1``  B=1  H=2  S=128   D=64  fp16 non-causal           seed 0
* ``c2``  packed qkv [B=2, S=512, 3, H=12, D=64] fp16 non-causal  seed 1
  ([P1] "实战集成" usage snippet: ``flash_attn_qkvpacked_func`` on [B,S,3,H,D])
* ``c3``  B=2  H=12 S=2048  D=64  fp16 causal / non-causal  seed 2
  ([P2] "实战代码对比" snippet: B=2, S=2048, 12 heads, head_dim 64)
* ``c3r`` as c3 with S=2000 (a ragged tail; not a multiple of 64)
* ``c4``  B=1  H=8  S=8192  D=128 bf16 causal               seed 3
  ([P4] §3.2: batch 1, 8 heads, sequence 8192, block 128 -> 512 blocks)
* ``c5``  B=1  H=16 S=16384 D=128 bf16 causal / non-causal  seed 4, Q and K
  drawn N(0, 2^2) to widen the softmax range

The e4m3 forward takes a workload's fp32 draws (same recipe, dtype ignored)
through ``quantize_e4m3``: one descale per tensor, max |x| mapped to 448.

Draw recipe: ``torch.Generator('cpu').manual_seed(seed)``; ``torch.randn`` in
fp32, in the order Q, K, V, dO (packed: qkv then dO); multiply Q and K by
``qk_std``; cast to the workload dtype. All tensors are [B, S, H, D].

Page legend: [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练";
[P2] "使用FlashAttention优化PyTorch模型注意力计算"; [P4] the FlashAttention-2
walkthrough published under the title "企业官网建设流程全解析".
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    dtype: torch.dtype
    causal: tuple
    seed: int
    packed: bool = False
    qk_std: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def fwd_flops(self, causal: bool) -> float:
        """Dense-contraction FLOPs of the forward: 4*B*H*Sq*Sk*D, halved if causal."""
        f = 4.0 * self.B * self.H * self.S * self.S * self.D
        return f / 2 if causal else f

    def bwd_flops(self, causal: bool) -> float:
        """Backward FLOPs by the 5-vs-2 matmul convention: 2.5x the forward."""
        return 2.5 * self.fwd_flops(causal)


WORKLOADS = {
    "c1": Workload("c1", 1, 2, 128, 64, torch.float16, (False,), 0),
    "c2": Workload("c2", 2, 12, 512, 64, torch.float16, (False,), 1, packed=True),
    "c3": Workload("c3", 2, 12, 2048, 64, torch.float16, (False, True), 2),
    "c3r": Workload("c3r", 2, 12, 2000, 64, torch.float16, (False, True), 2),
    "c4": Workload("c4", 1, 8, 8192, 128, torch.bfloat16, (True,), 3),
    "c5": Workload("c5", 1, 16, 16384, 128, torch.bfloat16, (False, True), 4, qk_std=2.0),
}


def draw(shape, seed_or_gen, dtype, std=1.0):
    """One N(0, std^2) tensor drawn in fp32 on the CPU and cast to ``dtype``."""
    g = seed_or_gen
    if not isinstance(g, torch.Generator):
        g = torch.Generator("cpu").manual_seed(int(seed_or_gen))
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def make_inputs(w: Workload, S: int | None = None, B: int | None = None, H: int | None = None):
    """Host tensors for workload ``w``: dict with q, k, v, do (and qkv if packed).

    ``S``, ``B`` and ``H`` override the workload sizes for smaller test cases
    that keep its dtype, seed and distribution.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    S = w.S if S is None else S
    g = torch.Generator("cpu").manual_seed(w.seed)
    out = {}
    if w.packed:
        qkv = torch.randn((B, S, 3, H, w.D), generator=g, dtype=torch.float32)
        qkv[:, :, 0:2] *= w.qk_std
        qkv = qkv.to(w.dtype)
        out["qkv"] = qkv
        out["q"], out["k"], out["v"] = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    else:
        for name, std in (("q", w.qk_std), ("k", w.qk_std), ("v", 1.0)):
            out[name] = draw((B, S, H, w.D), g, w.dtype, std)
    out["do"] = draw((B, S, H, w.D), g, w.dtype)
    return out


def random_case(B, H, Sq, Sk, D, dtype, seed, qk_std=1.0):
    """q [B,Sq,H,D], k/v [B,Sk,H,D], do [B,Sq,H,D] for ad-hoc shapes."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = draw((B, Sq, H, D), g, dtype, qk_std)
    k = draw((B, Sk, H, D), g, dtype, qk_std)
    v = draw((B, Sk, H, D), g, dtype)
    do = draw((B, Sq, H, D), g, dtype)
    return {"q": q, "k": k, "v": v, "do": do}


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor E4M3 encoding for the e4m3 forward's inputs: returns (bytes
    as a torch.uint8 tensor, descale) with x ~= value(bytes) * descale, the
    descale (an fp32 number) chosen so that max |x| lands on 448, the largest
    finite E4M3 value. The rounding is torch's float8_e4m3fn cast. This
    prepares inputs; it is not a step of the attention."""
    xf = x.float()
    amax = float(xf.abs().max()) if xf.numel() else 0.0
    descale = float(torch.tensor(amax / 448.0 if amax > 0 else 1.0, dtype=torch.float32))
    y = (xf / descale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return y.view(torch.uint8), descale


def make_e4m3_inputs(w: Workload, B: int | None = None, seed: int | None = None):
    """E4M3 inputs of workload ``w``'s shape: Q, K, V drawn as ``make_inputs``
    draws them (fp32, same order and seed, Q and K times ``qk_std``), then
    encoded by ``quantize_e4m3``. Returns {"q": (bytes, descale), "k": ..., "v": ...}."""
    B = w.B if B is None else B
    g = torch.Generator("cpu").manual_seed(w.seed if seed is None else seed)
    out = {}
    for name, std in (("q", w.qk_std), ("k", w.qk_std), ("v", 1.0)):
        out[name] = quantize_e4m3(draw((B, w.S, w.H, w.D), g, torch.float32, std))
    return out


def sample_rows(S: int, block: int, n_random: int, seed: int):
    """Query rows checked at full size: tile edges, the middle, the tail, plus
    ``n_random`` rows drawn with ``seed``. Sorted, unique."""
    fixed = [0, 1, block - 1, block, block + 1, S // 2, S - block - 1, S - block, S - 2, S - 1]
    g = torch.Generator("cpu").manual_seed(seed)
    rnd = torch.randint(0, S, (n_random,), generator=g).tolist()
    return sorted({r for r in fixed + rnd if 0 <= r < S})
