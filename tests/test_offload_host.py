"""Host side of the offload pipeline: how a layer is packed (no GPU)."""
import numpy as np
import pytest
import torch

import workloads
import huffman_decode_df11_b200 as df11
from huffman_decode_df11_b200 import offload


def test_packed_layout_is_aligned_and_complete(monkeypatch):
    # the decode table comes from the device; stand in a recognisable one
    monkeypatch.setattr(offload, "_tables_for",
                        lambda h, device: np.full(df11.DF11_DECODE_TABLE_BYTES, 7, np.uint8))
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    hs = [df11.compress(workloads.gaussian_bf16(n, 0.02, n)) for n in (1, 999, 100_003)]
    layer = offload.pack_layer(hs, device="cpu")
    flat = layer.host.numpy()
    spans = []
    for h, off in zip(hs, layer.offsets):
        for f in ("bitstream", "gaps", "chunk_counts", "block_out_pos", "luts",
                  "code_lengths", "sign_mantissa", "decode_table"):
            o, nbytes = off[f]
            assert o % 16 == 0
            spans.append((o, o + nbytes))
            if f == "decode_table":
                assert (flat[o:o + nbytes] == 7).all()
            else:
                want = np.ascontiguousarray(getattr(h, f)).view(np.uint8)
                assert nbytes == want.nbytes and np.array_equal(flat[o:o + nbytes], want)
    spans.sort()
    for (b0, e0), (b1, _) in zip(spans, spans[1:]):
        assert e0 <= b1           # no overlap
    assert spans[-1][1] <= layer.nbytes
    assert layer.n == [1, 999, 100_003]
