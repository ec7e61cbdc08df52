"""Decoding weights kept in host memory: the CPU-offload pattern.

The pages offload compressed weights to CPU memory when the GPU holds too
little, bringing each block's weights over as it is needed
("DFloat11无损压缩技术：基于哈夫曼编码的BFloat16大模型显存优化方案" §4.3;
"DFloat11：用于高效 GPU 推理的 LLM 和扩散模型无损压缩" "最新消息").

Here every layer (a group of compressed tensors) is packed into one pinned
host buffer: all its tensors' format buffers and decode tables, each at a
16-byte aligned offset.  Two device slots of the largest packed size take
the layers in turn.  For layer i:
- a copy stream waits until slot i % 2 is free (layer i-2's decode is done
  with it) and copies the packed layer into it (one host-to-device copy);
- the compute stream waits for that copy and decodes the layer from the slot
  into the caller's output buffers (one library call).
Layer i+1's copy then overlaps layer i's decode, and whatever the caller
queues after the decode on the compute stream (the layer's matmuls).  What
crosses PCIe is the compressed size, not the 2 bytes per weight of BF16.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

import numpy as np
import torch

from . import (DF11_DECODE_TABLE_BYTES, DecodePlan, Df11Device, Df11Host, Params,
               build_decode_table, to_device)

_FIELDS = ("bitstream", "gaps", "chunk_counts", "block_out_pos", "luts", "code_lengths",
           "sign_mantissa")


def _align16(x: int) -> int:
    return (x + 15) & ~15


@dataclass
class PackedLayer:
    """One layer's compressed tensors in one pinned host buffer."""
    host: torch.Tensor              # uint8, pinned
    offsets: List[dict]             # per tensor: field -> (offset, bytes)
    params: List[Params]
    shapes: List[tuple]

    @property
    def nbytes(self) -> int:
        return int(self.host.numel())

    @property
    def n(self) -> List[int]:
        return [int(p.n) for p in self.params]


def _tables_for(h: Df11Host, device) -> np.ndarray:
    """A tensor's decode table, derived once on the device and kept on the
    host with the rest of the layer."""
    d = to_device(h, device, decode_table=False)
    return build_decode_table(d).cpu().numpy()


def pack_layer(tensors: Sequence[Df11Host], device="cuda") -> PackedLayer:
    """Pack a layer's compressed tensors (and their decode tables) into one
    pinned host buffer."""
    arrays, offsets, pos = [], [], 0
    for h in tensors:
        table = _tables_for(h, device) if h.n else np.zeros(DF11_DECODE_TABLE_BYTES, np.uint8)
        fields = {f: np.ascontiguousarray(getattr(h, f)).view(np.uint8) for f in _FIELDS}
        fields["decode_table"] = table
        off = {}
        for f, a in fields.items():
            off[f] = (pos, a.nbytes)
            arrays.append((pos, a))
            pos = _align16(pos + a.nbytes)
        offsets.append(off)
    host = torch.empty(max(pos, 16), dtype=torch.uint8).pin_memory()
    flat = host.numpy()
    for p, a in arrays:
        flat[p:p + a.nbytes] = a
    return PackedLayer(host=host, offsets=offsets,
                       params=[Params.from_buffer_copy(h.params) for h in tensors],
                       shapes=[tuple(h.shape) for h in tensors])


def _device_views(layer: PackedLayer, slot: torch.Tensor) -> List[Df11Device]:
    """Df11Device views of a packed layer once it sits in `slot`."""
    out = []
    for off, p, shape in zip(layer.offsets, layer.params, layer.shapes):
        def view(f, dtype=torch.uint8):
            o, nbytes = off[f]
            t = slot[o:o + nbytes]
            return t.view(dtype) if dtype != torch.uint8 else t
        out.append(Df11Device(params=p, bitstream=view("bitstream"), gaps=view("gaps"),
                              block_out_pos=view("block_out_pos", torch.int32),
                              luts=view("luts", torch.int32),
                              code_lengths=view("code_lengths"),
                              sign_mantissa=view("sign_mantissa"),
                              chunk_counts=view("chunk_counts"), shape=shape,
                              decode_table=view("decode_table")))
    return out


class OffloadPipeline:
    """Decode layers kept in pinned host memory, one after another, with
    each layer's host-to-device copy overlapping the previous layer's
    decode.  `outs[i]` are the caller's device buffers for layer i's tensors
    (n 2-byte elements each, 16-byte aligned; one scratch buffer may serve
    every layer, since layer i+1's decode follows layer i's on the compute
    stream)."""

    def __init__(self, layers: Sequence[PackedLayer], outs: Sequence[Sequence[torch.Tensor]],
                 device="cuda"):
        if len(layers) != len(outs):
            raise ValueError("one output list per layer")
        self.layers = list(layers)
        self.device = torch.device(device)
        size = max(l.nbytes for l in self.layers)
        self.slots = [torch.empty(size, dtype=torch.uint8, device=self.device) for _ in range(2)]
        self.copy_stream = torch.cuda.Stream(self.device)
        # one decode plan per (layer, slot): descriptors point into the slot
        self.plans = [[DecodePlan(_device_views(l, s), o) for s in self.slots]
                      for l, o in zip(self.layers, outs)]
        self.copied = [torch.cuda.Event() for _ in self.layers]
        self.freed = [torch.cuda.Event() for _ in self.slots]
        self.h2d_bytes = sum(l.nbytes for l in self.layers)

    def run(self, err=None, stream=None, after_layer=None):
        """Copy and decode every layer once.  `after_layer(i)`, if given, is
        called after layer i's decode is queued on the compute stream (to
        queue that layer's use of the outputs there)."""
        compute = stream or torch.cuda.current_stream(self.device)
        # slots start free once the compute stream reaches this point
        for e in self.freed:
            e.record(compute)
        for i, layer in enumerate(self.layers):
            s = i % 2
            with torch.cuda.stream(self.copy_stream):
                self.copy_stream.wait_event(self.freed[s])
                self.slots[s][: layer.nbytes].copy_(layer.host, non_blocking=True)
                self.copied[i].record(self.copy_stream)
            compute.wait_event(self.copied[i])
            self.plans[i][s].run(err=err, stream=compute)
            self.freed[s].record(compute)  # the slot is read only by the decode
            if after_layer is not None:
                after_layer(i)
