"""autograd wrappers (flash_attn_func / flash_attn_qkvpacked_func) on the GPU:
gradients through loss.backward() against the fp64 oracle, and peak device
memory against attention that materialises the S x S score matrix."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_96_b200.autograd import PackedQKVAttention, flash_attn_func, flash_attn_qkvpacked_func
from exact_io_aware_96_b200.inputs import WORKLOADS, make_inputs, random_case
from tests.parity import check_grad, check_o_lse, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D,dtype", [(64, torch.float16), (128, torch.bfloat16)])
def test_flash_attn_func_backward(causal, D, dtype):
    c = random_case(2, 3, 333, 333, D, dtype, 77)
    q, k, v = (c[n].cuda().requires_grad_() for n in ("q", "k", "v"))
    do = c["do"].cuda()
    o = flash_attn_func(q, k, v, causal=causal)
    (o.float() * do.float()).sum().backward()
    sc = D ** -0.5
    o_ref, _ = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), sc, causal)
    assert np.max(np.abs(np64(o) - o_ref)) <= (1e-2 if dtype == torch.float16 else 2e-2)
    dq_r, dk_r, dv_r, _ = oracle.attention_backward(np64(c["q"]), np64(c["k"]), np64(c["v"]), np64(c["do"]), sc, causal)
    for g, r, name in ((q.grad, dq_r, "dq"), (k.grad, dk_r, "dk"), (v.grad, dv_r, "dv")):
        check_grad(np64(g), r, name, row_axis=1, head_axes=(0, 2))


def test_qkvpacked_usage_snippet():
    """The packed usage of the pages: qkv [B=2, S=512, 3, H=12, D=64] fp16,
    out = f(qkv) with shape [B, S, H, D], out.sum().backward()."""
    w = WORKLOADS["c2"]
    inp = make_inputs(w)
    qkv = inp["qkv"].cuda().requires_grad_()
    out = flash_attn_qkvpacked_func(qkv)
    assert tuple(out.shape) == (2, 512, 12, 64)
    out.sum().backward()
    assert qkv.grad is not None and tuple(qkv.grad.shape) == tuple(qkv.shape)
    qn, kn, vn = np64(inp["q"]), np64(inp["k"]), np64(inp["v"])
    ones = np.ones_like(qn)
    o_ref, _ = oracle.attention_forward(qn, kn, vn, w.scale, False)
    assert np.max(np.abs(np64(out) - o_ref)) <= 1e-2
    dq_r, dk_r, dv_r, _ = oracle.attention_backward(qn, kn, vn, ones, w.scale, False)
    g = np64(qkv.grad)
    for j, r in enumerate((dq_r, dk_r, dv_r)):
        check_grad(g[:, :, j], r, f"dqkv[{j}]", row_axis=1, head_axes=(0, 2))


def test_module_and_noncontiguous_inputs():
    c = random_case(1, 2, 200, 200, 64, torch.float16, 5)
    # [B, H, S, D] tensors transposed to [B, S, H, D] views: copied before the kernels see them
    q, k, v = (c[n].transpose(1, 2).contiguous().transpose(1, 2).cuda() for n in ("q", "k", "v"))
    o = flash_attn_func(q, k, v, causal=True)
    o_ref, _ = oracle.attention_forward(np64(c["q"]), np64(c["k"]), np64(c["v"]), 64 ** -0.5, True)
    assert np.max(np.abs(np64(o) - o_ref)) <= 1e-2
    qkv = torch.stack([c["q"], c["k"], c["v"]], dim=2).cuda()
    o2 = PackedQKVAttention(causal=True)(qkv)
    assert np.max(np.abs(np64(o2) - o_ref)) <= 1e-2


def _peak_bytes(fn):
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    fn()
    torch.cuda.synchronize()
    return torch.cuda.max_memory_allocated() - base


def _materialised(q, k, v, do, causal):
    """Standard attention through device memory: scores and probabilities
    stored as [B, H, S, S] tensors, autograd for the backward."""
    qh, kh, vh = (t.transpose(1, 2).detach().requires_grad_() for t in (q, k, v))
    s = (qh @ kh.transpose(-1, -2)) * (q.shape[-1] ** -0.5)
    if causal:
        S = s.shape[-1]
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool, device=s.device).triu(1), float("-inf"))
    p = torch.softmax(s, dim=-1)
    o = p @ vh
    o.backward(do.transpose(1, 2))


def _flash(q, k, v, do, causal):
    qq, kk, vv = (t.detach().requires_grad_() for t in (q, k, v))
    o = flash_attn_func(qq, kk, vv, causal=causal)
    o.backward(do)


@pytest.mark.parametrize("B,H,S,D,causal", [(2, 12, 2048, 64, False), (1, 8, 16384, 64, False)])
def test_peak_memory_linear_in_sequence(B, H, S, D, causal):
    """Forward + backward peak device memory beyond the inputs: the fused path
    keeps no S x S tensor, the materialised one holds several."""
    c = random_case(B, H, S, S, D, torch.float16, 3)
    q, k, v, do = (c[n].cuda() for n in ("q", "k", "v", "do"))
    flash = _peak_bytes(lambda: _flash(q, k, v, do, causal))
    mat = _peak_bytes(lambda: _materialised(q, k, v, do, causal))
    io = 4 * q.numel() * q.element_size()
    print(f"\npeak extra memory B{B} H{H} S{S} D{D}: fused {flash / 2**20:.1f} MiB, "
          f"materialised {mat / 2**20:.1f} MiB, ratio {mat / flash:.1f}x (inputs {io / 2**20:.1f} MiB)")
    assert flash < 8 * io                     # O(S): outputs, gradients, workspace
    assert mat > 2 * B * H * S * S * 2        # at least two S x S fp16 tensors
    assert mat > 4 * flash


def test_flash_attn_func_deterministic():
    c = random_case(1, 2, 300, 300, 128, torch.bfloat16, 91)
    grads = []
    for _ in range(2):
        q, k, v = (c[n].cuda().requires_grad_() for n in ("q", "k", "v"))
        flash_attn_func(q, k, v, causal=True, deterministic=True).backward(c["do"].cuda())
        grads.append((q.grad, k.grad, v.grad))
    for a, b in zip(*grads):
        assert torch.equal(a, b)
    dq_r, _, _, _ = oracle.attention_backward(np64(c["q"]), np64(c["k"]), np64(c["v"]), np64(c["do"]),
                                              128 ** -0.5, True)
    check_grad(np64(grads[0][0]), dq_r, "dq", row_axis=1, head_axes=(0, 2))
