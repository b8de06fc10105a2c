"""CUDA graphs of a step, specialised on whether the batch has any LoRA token.

"[LoRA] LoRA cuda graph specialization" (vllm-project/vllm pull 25914),
Implementation list: the batch descriptor gains a has_lora flag, two sets of
graphs are captured (one with the LoRA kernels, one without), and a batch in
which no token has an adapter replays the set without them.  LoRA being
enabled then costs an idle batch nothing on the device; the page's latency
logs put the cost without this at 10.5 % and with it at 1.4 %.

This module is that dispatch for a caller that captures its own step: the
step function enqueues the base work and, when asked, its LoRA calls through
this library; torch supplies the graphs.  The library's own no-active
short-circuit (has_active = 0 enqueues nothing) covers eager calls; inside a
captured graph the flag is fixed at capture time, which is why the two graph
sets are needed.
"""
from typing import Callable, Dict

import torch

from . import ops


class LoraGraphSet:
    """Two captured graphs of one step: has_lora False (no LoRA call at all)
    and True (the step's LoRA calls recorded).

        gs = LoraGraphSet(step).capture()
        gs.replay_for(idx_host, S)     # picks the graph from the batch's indices

    step(has_lora) enqueues one step on the current stream; with has_lora
    False it must enqueue no call of this library.  Inputs and outputs live
    in tensors the step closes over, so a replay reads whatever they hold.
    """

    def __init__(self, step: Callable[[bool], None], stream=None):
        self.step = step
        self.stream = stream if stream is not None else torch.cuda.Stream()
        self.graphs: Dict[bool, torch.cuda.CUDAGraph] = {}
        # library kernels recorded into each graph (lora_launch_count across
        # the capture): 0 for the graph without LoRA
        self.lora_launches: Dict[bool, int] = {}

    def capture(self, keep_graph: bool = False) -> "LoraGraphSet":
        for has_lora in (False, True):
            # one eager run first: kernel attributes and library workspaces are
            # set up outside the capture
            with torch.cuda.stream(self.stream):
                self.step(has_lora)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph(keep_graph=keep_graph)
            before = ops.launch_count()
            with torch.cuda.graph(g, stream=self.stream):
                self.step(has_lora)
            self.lora_launches[has_lora] = ops.launch_count() - before
            if keep_graph:
                g.instantiate()
            self.graphs[has_lora] = g
        return self

    def replay(self, has_lora: bool) -> None:
        self.graphs[bool(has_lora)].replay()

    def replay_for(self, idx_host, S: int) -> bool:
        """Replay the graph this batch needs: the one with LoRA kernels only
        when some index of the host copy selects a slot in [0, S).  Returns
        the flag used."""
        has = ops.active_from_host(idx_host, S)
        self.replay(has)
        return has
