"""Serving loop over a layer: host batches in, host outputs out.

``StepPipeline`` runs consecutive layer steps whose inputs arrive in pinned
host memory and whose outputs go back to pinned host memory, with the copies
of neighbouring steps overlapping the compute of the current one:

    copy stream:  H2D(i+1) -> staging[(i+1)%2]         D2H(i-1) <- out_stage[(i-1)%2]
    main stream:  graph[i%2]: staging[i%2] -> layer inputs, layer step, layer.out -> out_stage[i%2]

Each of the two graphs holds one device-to-device copy of the inputs from its
staging buffer, the whole layer step (``layer.forward``, both streams) and one
copy of the output to its staging buffer; events order a staging buffer's
refill after the step that read it and its D2H after the step that wrote it.
PyTorch provides the buffers, streams, events and graphs; every step of the
layer runs in ``libmoe_b200.so``.
"""
from __future__ import annotations

import torch


class StepPipeline:
    """Pipelined steps of ``layer`` (a ``MoELayer`` or ``FusedSharedMoELayer``).

    ``input_names``: the keys of ``layer.inp`` that change from step to step
    (e.g. ``("x", "logits")``); every step copies them in from the host.
    """

    def __init__(self, layer, input_names, stream=None):
        self.layer = layer
        self.names = list(input_names)
        dev = layer.device
        self.main = stream or torch.cuda.Stream(device=dev)
        self.copy = torch.cuda.Stream(device=dev)
        inp = layer.inp
        self.stage_in = [[torch.empty_like(inp[n]) for n in self.names] for _ in range(2)]
        self.stage_out = [torch.empty_like(layer.out) for _ in range(2)]
        self.ev_in = [torch.cuda.Event() for _ in range(2)]    # H2D into staging b done
        self.ev_step = [torch.cuda.Event() for _ in range(2)]  # step on buffers b done (inputs read, output staged)
        self.ev_d2h = [torch.cuda.Event() for _ in range(2)]   # D2H from out_stage b done
        self.graphs = []
        self.main.wait_stream(torch.cuda.current_stream(dev))
        for b in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(self.main):
                with torch.cuda.graph(g, stream=self.main):
                    for n, src in zip(self.names, self.stage_in[b]):
                        inp[n].copy_(src)
                    layer.forward(self.main)
                    self.stage_out[b].copy_(layer.out)
            self.graphs.append(g)
        torch.cuda.synchronize(dev)

    def run(self, host_inputs, host_outputs):
        """Enqueue len(host_inputs) steps. host_inputs[i]: pinned CPU tensors
        in ``input_names`` order; host_outputs[i]: a pinned CPU tensor shaped
        like ``layer.out``. Returns an event on the main stream that completes
        when the last output has reached the host."""
        n = len(host_inputs)
        if n == 0:
            ev = torch.cuda.Event()
            ev.record(self.main)
            return ev
        self.copy.wait_stream(self.main)  # after the caller's work on the main stream
        with torch.cuda.stream(self.copy):
            for dst, src in zip(self.stage_in[0], host_inputs[0]):
                dst.copy_(src, non_blocking=True)
            self.ev_in[0].record(self.copy)
        for i in range(n):
            b = i % 2
            # step i on the main stream: its inputs are staged, and the D2H of
            # step i - 2 (same output staging buffer) has drained
            self.main.wait_event(self.ev_in[b])
            if i >= 2:
                self.main.wait_event(self.ev_d2h[b])
            with torch.cuda.stream(self.main):
                self.graphs[b].replay()
            self.ev_step[b].record(self.main)
            with torch.cuda.stream(self.copy):
                if i + 1 < n:  # inputs of step i + 1, once step i - 1 is done with that buffer
                    nb = (i + 1) % 2
                    if i >= 1:
                        self.copy.wait_event(self.ev_step[nb])
                    for dst, src in zip(self.stage_in[nb], host_inputs[i + 1]):
                        dst.copy_(src, non_blocking=True)
                    self.ev_in[nb].record(self.copy)
                self.copy.wait_event(self.ev_step[b])
                host_outputs[i].copy_(self.stage_out[b], non_blocking=True)
                self.ev_d2h[b].record(self.copy)
        self.main.wait_event(self.ev_d2h[(n - 1) % 2])
        done = torch.cuda.Event()
        done.record(self.main)
        return done
