"""Attention forward + backward on batches that live in host memory.

``HostAttentionPipeline`` takes q, k, v and dO in pinned host memory, copies
them to the device, runs ``fa_fwd`` and ``fa_bwd`` through the C ABI, and
copies O, LSE, dQ, dK and dV back into pinned host memory. The copies of one
step overlap the kernels of its neighbours: host-to-device copies run on one
stream, the kernels on a second, device-to-host copies on a third, and the
device tensors come in ``depth`` sets used in turn, so step k+1's inputs
travel over PCIe while step k computes and step k-1's results travel back.
Every byte of every step still crosses the bus; nothing is cached between
steps. torch is used for device memory, streams, events and the copies; all
arithmetic runs in libfa.so.
"""
from __future__ import annotations

import torch

from . import fa


class HostAttentionPipeline:
    """Pipelined host-to-host attention steps of one fixed shape.

    ``step(...)`` enqueues one step and returns at once; ``synchronize()``
    waits for every enqueued step. Host tensors must be pinned, contiguous
    [B, S, H, D] (q, k, v, do, o, dq, dk, dv) and [B, H, S] fp32 (lse), and
    must not be reused for another step's outputs before that step is done.
    """

    def __init__(self, B, S, H, D, dtype=torch.bfloat16, causal=False, scale=None, device=None, depth=2,
                 deterministic=False):
        if not torch.cuda.is_available():
            raise RuntimeError("HostAttentionPipeline needs a CUDA device (the library has no CPU path)")
        self.shape = (B, S, H, D)
        self.dtype, self.causal, self.deterministic = dtype, bool(causal), bool(deterministic)
        self.scale = D ** -0.5 if scale is None else float(scale)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.depth = int(depth)
        if self.depth < 1:
            raise ValueError("depth must be >= 1")
        fa.lib()  # fail loudly if the library is missing
        mk = lambda: torch.empty(self.shape, dtype=dtype, device=self.device)  # noqa: E731
        self.sets = []
        for _ in range(self.depth):
            self.sets.append({
                "q": mk(), "k": mk(), "v": mk(), "do": mk(), "o": mk(), "dq": mk(), "dk": mk(), "dv": mk(),
                "lse": torch.empty((B, H, S), dtype=torch.float32, device=self.device),
                "ws": fa.workspace_for(B, H, S, D, self.device, Sk=S, deterministic=self.deterministic),
                "fws": fa.fwd_workspace_for(B, H, S, S, D, causal, self.device),
                # compute done with this set's inputs / forward outputs ready / results copied out
                "computed": torch.cuda.Event(), "fwd_done": torch.cuda.Event(), "copied_out": torch.cuda.Event(),
                "copied_in": torch.cuda.Event(), "used": False,
            })
        self.s_in = torch.cuda.Stream(self.device)
        self.s_comp = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)
        self.k = 0

    def _check(self, name, t, shape, dtype):
        if t.device.type != "cpu" or not t.is_pinned() or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous pinned host tensor")
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
            raise ValueError(f"{name}: expected {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")

    def step(self, hq, hk, hv, hdo, ho, hlse, hdq, hdk, hdv):
        """Enqueue one step: inputs hq, hk, hv, hdo; outputs ho, hlse, hdq, hdk, hdv."""
        B, S, H, D = self.shape
        for name, t in (("q", hq), ("k", hk), ("v", hv), ("do", hdo), ("o", ho), ("dq", hdq), ("dk", hdk),
                        ("dv", hdv)):
            self._check(name, t, self.shape, self.dtype)
        self._check("lse", hlse, (B, H, S), torch.float32)
        st = self.sets[self.k % self.depth]
        self.k += 1
        with torch.cuda.stream(self.s_in):
            if st["used"]:
                self.s_in.wait_event(st["computed"])        # the kernels are done with these inputs
            for src, name in ((hq, "q"), (hk, "k"), (hv, "v"), (hdo, "do")):
                st[name].copy_(src, non_blocking=True)
            st["copied_in"].record(self.s_in)
        with torch.cuda.stream(self.s_comp):
            self.s_comp.wait_event(st["copied_in"])
            if st["used"]:
                self.s_comp.wait_event(st["copied_out"])    # the previous results left the device
            fa.forward(st["q"], st["k"], st["v"], causal=self.causal, scale=self.scale, out=st["o"],
                       lse=st["lse"], stream=self.s_comp, workspace=st["fws"],
                       split_ranks=0 if st["fws"] is not None else -1)
            st["fwd_done"].record(self.s_comp)
            fa.backward(st["q"], st["k"], st["v"], st["o"], st["lse"], st["do"], causal=self.causal,
                        scale=self.scale, dq=st["dq"], dk=st["dk"], dv=st["dv"], workspace=st["ws"],
                        stream=self.s_comp, deterministic=self.deterministic)
            st["computed"].record(self.s_comp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(st["fwd_done"])
            ho.copy_(st["o"], non_blocking=True)
            hlse.copy_(st["lse"], non_blocking=True)
            self.s_out.wait_event(st["computed"])
            for dst, name in ((hdq, "dq"), (hdk, "dk"), (hdv, "dv")):
                dst.copy_(st[name], non_blocking=True)
            st["copied_out"].record(self.s_out)
        st["used"] = True

    def join(self, stream=None):
        """Make `stream` (default: the current stream) wait for every enqueued step."""
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        for t in (self.s_in, self.s_comp, self.s_out):
            s.wait_stream(t)

    def start_after(self, stream=None):
        """Make the pipeline's streams wait for work already enqueued on `stream`."""
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        for t in (self.s_in, self.s_comp, self.s_out):
            t.wait_stream(s)

    def synchronize(self):
        for t in (self.s_in, self.s_comp, self.s_out):
            t.synchronize()

    @property
    def h2d_bytes_per_step(self):
        B, S, H, D = self.shape
        return 4 * B * S * H * D * torch.tensor([], dtype=self.dtype).element_size()

    @property
    def d2h_bytes_per_step(self):
        B, S, H, D = self.shape
        return 4 * B * S * H * D * torch.tensor([], dtype=self.dtype).element_size() + B * H * S * 4
