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


def test_device_tensor_in_one_block_views_and_pointers():
    """A device-built tensor keeps its buffers as byte ranges of one
    allocation (Df11Device._in_block): every buffer read as an attribute is
    that range, with the view the format gives it, and the pointers a decode
    takes come straight from the allocation, before and after a view is
    made.  Checked on a host tensor standing in for the allocation."""
    block = torch.arange(8192, dtype=torch.int32).view(torch.uint8)[:8192]
    offs = (0, 256, 512, 768, 1024, 2048, 2304)
    sizes = (40, 21, 32, 12, 1024, 256, 16)
    d = df11.Df11Device._in_block(df11.Params(), block, offs, sizes, (4, 4), 1)
    base = block.data_ptr()
    names = ("bitstream", "gaps", "chunk_counts", "block_out_pos", "luts", "code_lengths",
             "sign_mantissa")
    # pointers before any view exists
    for name, o in zip(names, offs):
        assert d._ptr(name) == base + o
    for name, o, nb in zip(names, offs, sizes):
        v = getattr(d, name)
        want = block[o:o + nb]
        if name in ("block_out_pos", "luts"):
            assert v.dtype == torch.int32 and v.numel() == nb // 4
            want = want.view(torch.int32)
        else:
            assert v.dtype == torch.uint8 and v.numel() == nb
        assert v.data_ptr() == base + o
        assert torch.equal(v, want)
        assert d._ptr(name) == base + o  # and after
    assert d.device == block.device and d.shape == (4, 4) and d.decode_table is None
    desc = d.desc(torch.empty(16, dtype=torch.bfloat16))
    assert desc.bitstream == base and desc.chunk_counts == base + offs[2]
    assert desc.sign_mantissa == base + offs[6]
    with pytest.raises(AttributeError):
        d.not_a_buffer


def test_device_tensor_built_the_usual_way_keeps_its_defaults():
    """The constructor still defaults chunk_counts to None (its class
    attribute is gone, so that a tensor in one block can make it lazily)."""
    t = torch.zeros(64, dtype=torch.uint8)
    d = df11.Df11Device(params=df11.Params(), bitstream=t, gaps=t, block_out_pos=t, luts=t,
                        code_lengths=t, sign_mantissa=t)
    assert d.chunk_counts is None and d.interleave == 1 and d.shape == ()
    desc = d.desc(torch.empty(16, dtype=torch.bfloat16))
    assert not desc.chunk_counts
