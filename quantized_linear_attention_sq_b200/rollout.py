"""Several layers' state pools stepped together, eagerly or as one CUDA graph.

A model's decode token runs the state step once per layer, so launching it
per layer costs the host L launches per token. ``LayerStack.capture``
records `steps` tokens x L layers of step launches into one CUDA graph that
reads its activations from fixed device buffers and writes fixed outputs;
one replay then issues all of them with a single host call. Every launch
still runs in libsq.so (the step allocates nothing and never synchronizes,
so it can be captured; each launch leaves its handle's work counter at
zero, so replays start from a clean counter).
"""
from __future__ import annotations

import torch

from .state import StatePool


class LayerStack:
    """L state pools (one StatePool handle per layer, each with its own
    calibration) stepped in layer order."""

    def __init__(self, layers: list[StatePool]):
        if not layers:
            raise ValueError("a LayerStack needs at least one layer")
        self.layers = list(layers)

    def __len__(self):
        return len(self.layers)

    def new_pools(self) -> list[torch.Tensor]:
        return [sp.new_pool() for sp in self.layers]

    def step(self, pools, inputs, outs, slot_ids=None, stream=None):
        """One token through every layer: inputs[l] = (q, k, v, beta, g),
        outs[l] the layer's o."""
        if not (len(pools) == len(inputs) == len(outs) == len(self.layers)):
            raise ValueError("pools, inputs and outs need one entry per layer")
        for sp, pool, x, o in zip(self.layers, pools, inputs, outs):
            sp.decode_step(pool, *x, o, slot_ids=slot_ids, stream=stream)

    def capture(self, pools, inputs_seq, outs_seq, slot_ids=None) -> torch.cuda.CUDAGraph:
        """Record len(inputs_seq) tokens x L layers of steps into one CUDA
        graph (nothing runs during the capture). inputs_seq[t][l] and
        outs_seq[t][l] are the device buffers the replay reads and writes;
        pools are updated in place by every replay."""
        if len(inputs_seq) != len(outs_seq) or not inputs_seq:
            raise ValueError("inputs_seq and outs_seq need the same, non-zero number of tokens")
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for x_t, o_t in zip(inputs_seq, outs_seq):
                    self.step(pools, x_t, o_t, slot_ids=slot_ids)
        torch.cuda.current_stream().wait_stream(side)
        return graph

    def close(self):
        for sp in self.layers:
            sp.close()
