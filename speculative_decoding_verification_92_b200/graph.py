"""Replay a whole verification step as one CUDA graph.

For small batches the step is bound by host launch work, not by the GPU. The
call marshals arguments through ctypes, checks them, and enqueues two kernel
launches with cluster and programmatic-dependent-launch attributes. Capturing
spec_verify once into a CUDA graph over fixed buffers turns every later step
into a single graph launch.

``VerifyGraph`` owns static device copies of the inputs, the outputs and the
workspace. Each step copies new inputs into the static buffers (or the caller
writes them there directly through ``.inputs``) and replays. The captured
launches are exactly spec_verify's kernels; nothing is re-implemented here.
"""
from __future__ import annotations

from . import spec_verify, workspace_bytes, BF16, F32


class VerifyGraph:
    """spec_verify captured once for fixed shapes, dtype, temperature and
    mode.

    Input tensors passed to the constructor fix the shapes.  Their data is
    copied into the graph's own buffers (``self.inputs``); ``step()`` takes
    new inputs of the same shapes (or None to reuse what the buffers hold),
    replays the graph on the current stream and returns the static output
    tensors ``(accept_len, tokens)``, which the next replay overwrites."""

    def __init__(self, target, draft, tokens, lens, uniforms, temperature=1.0, greedy=False, *, V=None):
        import torch
        self.torch = torch
        dev = target.device

        def own(t):
            return None if t is None else t.detach().clone()

        self.inputs = dict(target=own(target), draft=own(draft), tokens=own(tokens), lens=own(lens),
                           uniforms=own(uniforms))
        B, k = tokens.shape
        self.V = V if V is not None else target.shape[-1]
        dt = BF16 if target.dtype == torch.bfloat16 else F32
        row_stride = target.shape[-1]
        self.workspace = torch.empty(max(workspace_bytes(B, k, self.V, dt, row_stride), 256),
                                     dtype=torch.uint8, device=dev)
        self.out = (torch.empty(B, dtype=torch.int32, device=dev),
                    torch.empty(B, k + 1, dtype=torch.int32, device=dev))
        self.temperature, self.greedy = float(temperature), bool(greedy)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self._run(side)            # warm-up outside capture: kernel attributes, device caches
        side.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=side):
            self._run(side)
        torch.cuda.current_stream(dev).wait_stream(side)

    def _run(self, stream):
        i = self.inputs
        spec_verify(i["target"], None if self.greedy else i["draft"], i["tokens"], i["lens"],
                    None if self.greedy else i["uniforms"], self.temperature, self.greedy, V=self.V,
                    out=self.out, workspace=self.workspace, stream=stream)

    def step(self, target=None, draft=None, tokens=None, lens=None, uniforms=None):
        for name, t in (("target", target), ("draft", draft), ("tokens", tokens), ("lens", lens),
                        ("uniforms", uniforms)):
            if t is not None:
                self.inputs[name].copy_(t, non_blocking=True)
        self.graph.replay()
        return self.out
