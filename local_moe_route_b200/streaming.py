"""Host-resident expert weights streamed to the GPU while the previous layer
computes.

The engine the pages describe keeps most experts in host memory because a
12-24 GB card cannot hold them, processes prefill in 6144-token chunks so
that every expert crosses PCIe once per chunk instead of once per 512
tokens, and has a separate thread DMA the next layer's experts into a GPU
ring buffer so that layer N + 1's upload overlaps layer N's compute
(kongchang.com "两天移植，预填充提速8倍：Strata引擎实测", section "Strata快在哪";
the ported fork streams experts on a second CUDA stream, same page, next
section).  One B200 holds every expert of a layer, so this path matters only
for models whose experts exceed HBM.

`LayerStreamer` keeps the packed int4 weights and fp16 scales of every layer
in pinned host memory and `slots` device copies of one layer's weights (a
ring).  `forward` runs the layers in order on the compute stream; a copy
stream uploads layer i + slots - 1 into the slot that layer i - 1 used as
soon as that layer's forward has finished with it, so the upload of the
next layers overlaps the current layer's forward.  CUDA events order the
two streams; nothing synchronises the host.
"""

from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import torch

WEIGHTS = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")


class LayerStreamer:
    def __init__(self, layers: Sequence[Dict[str, torch.Tensor]], dims: dict, device,
                 slots: int = 2):
        """layers: per layer a dict with the six weight tensors (host, any
        memory; copied into pinned buffers once), `w_router` (bf16 bits) and
        optionally `bias`.  Router matrices stay on the device (4 MB each)."""
        import local_moe_route_b200 as sm
        if slots < 2:
            raise ValueError("a ring needs at least two slots to overlap")
        self.sm = sm
        self.dims = dict(dims)
        self.dev = torch.device(device)
        self.L = len(layers)
        self.slots = min(slots, self.L)
        self.host: List[Dict[str, torch.Tensor]] = []
        self.router: List[torch.Tensor] = []
        self.bias: List[Optional[torch.Tensor]] = []
        for lay in layers:
            self.host.append({n: lay[n].contiguous().pin_memory() for n in WEIGHTS})
            self.router.append(lay["w_router"].to(self.dev).view(torch.bfloat16))
            b = lay.get("bias")
            self.bias.append(None if b is None else b.to(self.dev))
        self.ring = [{n: torch.empty_like(self.host[0][n], device=self.dev) for n in WEIGHTS}
                     for _ in range(self.slots)]
        self.copy_stream = torch.cuda.Stream(device=self.dev)
        self.loaded = [torch.cuda.Event() for _ in range(self.slots)]
        self.freed = [torch.cuda.Event() for _ in range(self.slots)]
        self.bytes_per_layer = sum(t.numel() * t.element_size() for t in self.host[0].values())

    def _upload(self, layer: int, slot: int, compute: torch.cuda.Stream):
        with torch.cuda.stream(self.copy_stream):
            self.copy_stream.wait_event(self.freed[slot])
            for n in WEIGHTS:
                self.ring[slot][n].copy_(self.host[layer][n], non_blocking=True)
            self.loaded[slot].record(self.copy_stream)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, events: Optional[list] = None) -> torch.Tensor:
        """x [T][d] bf16 on the device through all layers; returns the last
        layer's output.  `events`, if given, receives (start, end) CUDA events
        of every layer's forward on the compute stream."""
        sm = self.sm
        compute = torch.cuda.current_stream(self.dev)
        T = x.shape[0]
        dims = dict(self.dims, T=T)
        ws = sm.workspace(dims, self.dev) if ws is None else ws
        bufs = [torch.empty_like(x), torch.empty_like(x)]
        for s in range(self.slots):
            self.freed[s].record(compute)
        for i in range(self.slots - 1):
            self._upload(i, i % self.slots, compute)
        cur = x
        for i in range(self.L):
            slot = i % self.slots
            nxt = i + self.slots - 1
            if nxt < self.L:
                self._upload(nxt, nxt % self.slots, compute)
            compute.wait_event(self.loaded[slot])
            w = self.ring[slot]
            out = y if (i == self.L - 1 and y is not None) else bufs[i & 1]
            e0 = torch.cuda.Event(enable_timing=True) if events is not None else None
            if e0 is not None:
                e0.record(compute)
            sm.check(sm.strata_moe_forward(cur, self.router[i], self.bias[i],
                                           (w["gate_q"], w["gate_s"]), (w["up_q"], w["up_s"]),
                                           (w["down_q"], w["down_s"]), dims, out, None, None, ws,
                                           stream=compute), f"layer {i}")
            if e0 is not None:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(compute)
                events.append((e0, e1))
            self.freed[slot].record(compute)
            cur = out
        return cur
