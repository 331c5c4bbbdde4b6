"""Block decode driver: the sub-block loop of one block on the device.

Block-wise decoding ("Fast-dLLM v2" Levels 1-3; technical review
Algorithm 1): a block of D positions starts fully masked; its sub-blocks are
decoded left to right, each by repeating a denoising step while any of its
positions is still masked; the finished block's K/V are then appended to the
prefix cache.  Here each sub-block's repetition is a CUDA-graph WHILE node
whose body is the caller's step (captured once) followed by
``fdl_unit_status``, which sets the node's condition from ``n_masked_left``
on the device.  A whole block is one graph launch with no host round trip.

``step(u, stream)`` must enqueue one denoising step of sub-block ``u`` on
``stream`` (a ``RawStream``, accepted by every ``fdl`` call; for example the
model's forward for the unit followed by ``fdl.denoise_step``); the driver
adds the loop control and the block append.  The host-loop variant (``run_host_loop``) reads the
``any_masked`` flag after each step instead, for comparison and debugging.
"""
from __future__ import annotations

import contextlib
from typing import Callable, List

import torch

from block_diffusion_decoding_causal_b200 import fdl


def _ck(res):
    err = res[0] if isinstance(res, tuple) else res
    if int(err) != 0:
        raise RuntimeError(f"CUDA runtime error {err}")
    if isinstance(res, tuple):
        return res[1] if len(res) == 2 else res[1:]
    return None


class RawStream:
    """A raw CUDA stream handle in the shape the fdl binding reads (it only
    uses ``cuda_stream``)."""

    def __init__(self, handle):
        self.cuda_stream = int(handle)


class BlockGraph:
    """One CUDA graph that decodes one block: per sub-block a WHILE node
    around (step, unit status), then the block-cache append.

    unit_cfgs: one fdl StepCfg per sub-block (q_off differs);
    n_masked_left: device int32 [B], written by each step's commit;
    steps: device int32 [n_units], step counter per sub-block (zeroed by the
      caller before a launch);
    append: callable(stream) enqueuing fdl_append_block, or None.
    """

    def __init__(self, unit_cfgs, step: Callable[[int, int], None], n_masked_left,
                 steps, append=None, max_iterations: int = 0):
        from cuda.bindings import runtime as rt
        self.rt = rt
        self.graph = _ck(rt.cudaGraphCreate(0))
        self._torch_stream = torch.cuda.Stream()
        self.stream = RawStream(self._torch_stream.cuda_stream)
        self._keep = []
        deps: List = []
        for u, cfg in enumerate(unit_cfgs):
            handle = _ck(rt.cudaGraphConditionalHandleCreate(
                self.graph, 1, rt.cudaGraphConditionalHandleFlags.cudaGraphCondAssignDefault))
            params = rt.cudaGraphNodeParams()
            params.type = rt.cudaGraphNodeType.cudaGraphNodeTypeConditional
            params.conditional.handle = handle
            params.conditional.type = rt.cudaGraphConditionalNodeType.cudaGraphCondTypeWhile
            params.conditional.size = 1
            node = _ck(rt.cudaGraphAddNode(self.graph, deps, len(deps), params))
            body = params.conditional.phGraph_out[0]
            s = self.stream.cuda_stream
            _ck(rt.cudaStreamBeginCaptureToGraph(
                s, body, None, None, 0,
                rt.cudaStreamCaptureMode.cudaStreamCaptureModeThreadLocal))
            with self._capturing(s):
                step(u, self.stream)
                fdl.unit_status(cfg, n_masked_left, None, steps[u:u + 1],
                                int(handle), stream=self.stream)
            self._keep.append((handle, params))
            deps = [node]
        if append is not None:
            s = self.stream.cuda_stream
            _ck(rt.cudaStreamBeginCaptureToGraph(
                s, self.graph, deps, None, len(deps),
                rt.cudaStreamCaptureMode.cudaStreamCaptureModeThreadLocal))
            with self._capturing(s):
                append(self.stream)
        self.exec = _ck(rt.cudaGraphInstantiate(self.graph, 0))

    @contextlib.contextmanager
    def _capturing(self, s):
        """End the capture on the way out, also when the body raised (a
        capture left open would make every later call on this thread fail)."""
        try:
            yield
        except BaseException:
            self.rt.cudaStreamEndCapture(s)
            raise
        _ck(self.rt.cudaStreamEndCapture(s))

    def launch(self, stream: torch.cuda.Stream = None):
        s = (stream or torch.cuda.current_stream()).cuda_stream
        _ck(self.rt.cudaGraphLaunch(self.exec, s))

    def __del__(self):
        try:
            self.rt.cudaGraphExecDestroy(self.exec)
            self.rt.cudaGraphDestroy(self.graph)
        except Exception:
            pass


def run_host_loop(unit_cfgs, step: Callable[[int, int], None], n_masked_left, any_masked,
                  steps_out: List[int], max_steps: int = 1024, stream=None):
    """The same loop driven from the host: after each step read the device
    flag written by fdl_unit_status (one synchronisation per step)."""
    s = stream or torch.cuda.current_stream()
    for u, cfg in enumerate(unit_cfgs):
        n = 0
        while True:
            step(u, s)
            fdl.unit_status(cfg, n_masked_left, any_masked, None, 0, stream=s)
            n += 1
            s.synchronize()
            if int(any_masked.item()) == 0 or n >= max_steps:
                break
        steps_out.append(n)
