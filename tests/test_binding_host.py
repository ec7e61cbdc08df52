"""Host-side pieces of the binding that need no GPU: the interleaved element
order (interleave_rows / deinterleave_rows) and the host builder's
`interleave` option, checked against explicit index loops and the oracle's
bit-serial decode."""
import numpy as np
import pytest
import torch

import oracle
import huffman_decode_df11_b200 as df11


def _loop_order(W, R):
    rows, cols = W.shape
    out = []
    for rb in range(rows // R):
        for cg in range(cols // 16):
            for r in range(R):
                out.extend(W[rb * R + r, cg * 16:(cg + 1) * 16])
    return np.array(out, dtype=W.dtype)


@pytest.mark.parametrize("rows,cols,R", [(8, 16, 8), (64, 48, 8), (32, 32, 32), (6, 64, 2),
                                         (5, 16, 1)])
def test_interleave_order_matches_the_definition(rows, cols, R):
    W = np.arange(rows * cols, dtype=np.uint16).reshape(rows, cols)
    flat = df11.interleave_rows(W, R)
    assert np.array_equal(flat, _loop_order(W, R))
    assert np.array_equal(df11.deinterleave_rows(flat, (rows, cols), R), W)
    t = torch.from_numpy(W.astype(np.int16))
    ft = df11.interleave_rows(t, R)
    assert np.array_equal(ft.numpy().view(np.uint16), flat)
    assert torch.equal(df11.deinterleave_rows(ft, (rows, cols), R), t)


@pytest.mark.parametrize("shape,R", [((12, 16), 8), ((16, 24), 8), ((16, 16), 3),
                                     ((256, 16), 256)])
def test_interleave_rejects_shapes_it_cannot_take(shape, R):
    with pytest.raises(ValueError):
        df11.interleave_rows(np.zeros(shape, np.uint16), R)


def test_host_builder_interleave_encodes_the_interleaved_order():
    rng = np.random.default_rng(4)
    W = (np.float32(rng.normal(0, 0.02, 64 * 96)).view(np.uint32) >> 16).astype(np.uint16)
    W = W.reshape(64, 96)
    h = df11.compress(W, 8, 128, interleave=8)
    assert h.interleave == 8 and h.shape == (64, 96)
    words, end, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, h.n)
    assert end == h.params.total_bits
    assert np.array_equal(words, _loop_order(W, 8))
