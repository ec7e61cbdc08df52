"""Fused decode and matrix-vector product (df11_decode_gemv) against the
oracle.

The oracle decodes the stream bit by bit and multiplies in float64
(oracle.gemv).  The GPU multiplies the decoded BF16 weights by BF16
activations in fp32: every product is exact in fp32 (8-bit significands),
and only the sums round.  For a sum of K terms in any order, each rounding
at most u = 2^-24 relative, the result is within gamma_K * sum |w x| of the
exact value, gamma_K = K u / (1 - K u) (the standard bound for recursive
summation in floating point).  Each output element is checked against
that bound with K = cols, computed from the oracle's own |W| |x|.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

df11 = pytest.importorskip("huffman_decode_df11_b200")

U32 = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _bound(h, cols, x_u16):
    """gamma_cols * (|W| |x|) per output, float64 (batch, rows)."""
    w, _, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, h.n)
    W = np.abs(oracle.bf16_to_f64(w)).reshape(-1, cols)
    X = np.abs(oracle.bf16_to_f64(x_u16)).reshape(-1, cols)
    g = cols * U32 / (1 - cols * U32)
    return g * (X @ W.T)


def _weights(rows, cols, seed, std=None):
    std = std if std is not None else 1.0 / np.sqrt(cols)
    return workloads.gaussian_bf16(rows * cols, std, seed).view(rows, cols)


def _acts(batch, cols, seed):
    return workloads.gaussian_bf16(batch * cols, 1.0, 10_000 + seed).view(batch, cols)


def _check(h, cols, x_bits, y_gpu, y0=None):
    xu = workloads.as_numpy_u16(x_bits)
    ref = oracle.gemv(h.bitstream, h.code_lengths, h.sign_mantissa, h.n, cols, xu)
    if y0 is not None:
        ref = ref + y0
    got = y_gpu.double().cpu().numpy().reshape(ref.shape)
    if y0 is None:
        bound = _bound(h, cols, xu)
    else:  # y0 is one more term of the sum
        k = cols + 1
        bound = (_bound(h, cols, xu) / (cols * U32 / (1 - cols * U32)) + np.abs(y0)) * \
            (k * U32 / (1 - k * U32))
    err = np.abs(got - ref)
    assert np.all(err <= bound), (float(err.max()), float(bound[err > bound].min()))


@pytest.mark.parametrize("rows,cols,batch,C", [
    (4096, 4096, 1, 24), (1024, 4096, 1, 24), (4096, 12288, 1, 24), (512, 4096, 4, 24),
    (1024, 4096, 8, 24), (768, 1024, 3, 16), (1000, 2048, 2, 8), (37, 48, 3, 24),
    (300, 16, 2, 24), (64, 400, 1, 24)])
def test_gemv_within_fp32_bound(rows, cols, batch, C):
    w = _weights(rows, cols, rows * 7 + cols + batch)
    h = df11.compress(workloads.as_numpy_u16(w), C, 256)
    h.shape = (rows, cols)
    d = df11.to_device(h, "cuda")
    x = _acts(batch, cols, rows + cols)
    y = torch.full((batch, rows), 123.0, dtype=torch.float32, device="cuda")
    err = df11.new_error_word()
    df11.decode_gemv([d], [x.cuda().view(torch.bfloat16)], [y], err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    _check(h, cols, x, y)


def test_accumulate_and_strides():
    rows, cols, batch = 777, 1024, 3
    w = _weights(rows, cols, 5)
    h = df11.compress(workloads.as_numpy_u16(w))
    h.shape = (rows, cols)
    d = df11.to_device(h, "cuda")
    xs = torch.zeros(batch, cols + 64, dtype=torch.int16)
    xs[:, :cols] = _acts(batch, cols, 3)
    x = xs.cuda()[:, :cols]                        # x_stride = cols + 64
    y0 = torch.randn(batch, rows + 5, dtype=torch.float64)
    ybuf = y0.float().cuda()
    y = ybuf[:, :rows]                             # y_stride = rows + 5
    df11.decode_gemv([d], [x.view(torch.bfloat16)], [y], accumulate=True)
    torch.cuda.synchronize()
    _check(h, cols, xs[:, :cols].contiguous(), y.contiguous(),
           y0=y0[:, :rows].float().double().numpy())
    assert torch.equal(ybuf[:, rows:].cpu(), y0[:, rows:].float())  # past the rows: untouched


def test_a_block_of_tensors_in_one_call():
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (12288, 4096),
              (12288, 4096), (4096, 12288)]
    hs, ds, xs, ys = [], [], [], []
    for i, (r, c) in enumerate(shapes):
        w = _weights(r, c, 40 + i)
        h = df11.compress(workloads.as_numpy_u16(w))
        h.shape = (r, c)
        hs.append(h)
        ds.append(df11.to_device(h, "cuda"))
        xs.append(_acts(1, c, 50 + i))
        ys.append(torch.empty(1, r, dtype=torch.float32, device="cuda"))
    err = df11.new_error_word()
    df11.decode_gemv(ds, [x.cuda().view(torch.bfloat16) for x in xs], ys, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for h, (r, c), x, y in zip(hs, shapes, xs, ys):
        _check(h, c, x, y)


def test_matches_decode_then_matmul_in_float64():
    rows, cols = 2048, 4096
    w = _weights(rows, cols, 11)
    h = df11.compress(workloads.as_numpy_u16(w))
    h.shape = (rows, cols)
    d = df11.to_device(h, "cuda")
    x = _acts(2, cols, 12).cuda()
    y = torch.empty(2, rows, dtype=torch.float32, device="cuda")
    df11.decode_gemv([d], [x.view(torch.bfloat16)], [y])
    W = df11.decode(d).view(rows, cols).double()
    ref = x.view(torch.bfloat16).double() @ W.T
    torch.cuda.synchronize()
    g = cols * U32 / (1 - cols * U32)
    bound = g * (x.view(torch.bfloat16).double().abs() @ W.abs().T)
    assert torch.all((y.double() - ref).abs() <= bound)


def test_argument_errors():
    w = _weights(64, 256, 1)
    h = df11.compress(workloads.as_numpy_u16(w))
    h.shape = (64, 256)
    d = df11.to_device(h, "cuda")
    x = _acts(1, 256, 1).cuda().view(torch.bfloat16)
    y = torch.empty(1, 64, dtype=torch.float32, device="cuda")
    L = df11.lib()
    desc = (df11.TensorDesc * 1)(d.desc(y))
    desc[0].out_bf16 = None

    def op(**kw):
        f = dict(x=x.data_ptr(), y=y.data_ptr(), cols=256, batch=1, x_stride=256, y_stride=64,
                 accumulate=0, pad=0)
        f.update(kw)
        return (df11.GemvOp * 1)(df11.GemvOp(**f))

    assert L.df11_decode_gemv(desc, op(), 1, None, None) == 0
    assert L.df11_decode_gemv(desc, op(cols=24), 1, None, None) == 7    # not a multiple of 16
    assert L.df11_decode_gemv(desc, op(cols=96), 1, None, None) == 7    # does not divide n
    assert L.df11_decode_gemv(desc, op(batch=9), 1, None, None) == 7
    assert L.df11_decode_gemv(desc, op(batch=0), 1, None, None) == 7
    assert L.df11_decode_gemv(desc, op(x_stride=260), 1, None, None) == 7
    assert L.df11_decode_gemv(desc, op(y_stride=63), 1, None, None) == 7
    assert L.df11_decode_gemv(desc, op(y=None), 1, None, None) == 1
    assert L.df11_decode_gemv(desc, op(x=x.data_ptr() + 8), 1, None, None) == 2
    desc[0].chunk_counts = None
    assert L.df11_decode_gemv(desc, op(), 1, None, None) == 4       # needs chunk counts
    torch.cuda.synchronize()
    with pytest.raises(ValueError):
        df11.decode_gemv([d], [x[:, :128]], [y])


def test_more_than_one_launch_and_both_modes():
    """20 weights in one call: the descriptor array is split into launches
    of at most 16 (product and clearing kernels alike); once adding into a
    given y, once clearing it first."""
    hs, ds, xs, y0s = [], [], [], []
    for i in range(20):
        rows, cols = 32 + 16 * i, 256 * (1 + i % 3)
        w = _weights(rows, cols, 200 + i)
        h = df11.compress(workloads.as_numpy_u16(w))
        h.shape = (rows, cols)
        hs.append(h)
        ds.append(df11.to_device(h, "cuda"))
        xs.append(_acts(2, cols, 300 + i))
        y0s.append(torch.randn(2, rows, dtype=torch.float64))
    xd = [x.cuda().view(torch.bfloat16) for x in xs]
    err = df11.new_error_word()
    ya = [y0.float().cuda() for y0 in y0s]
    df11.decode_gemv(ds, xd, ya, accumulate=True, err=err)
    yc = [torch.full_like(y, 7.0) for y in ya]
    df11.decode_gemv(ds, xd, yc, accumulate=False, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for h, x, y0, y_acc, y_clr in zip(hs, xs, y0s, ya, yc):
        cols = h.shape[1]
        _check(h, cols, x, y_acc, y0=y0.float().double().numpy())
        _check(h, cols, x, y_clr)


@pytest.mark.parametrize("rows,cols,batch,R", [
    (4096, 4096, 1, 8), (1024, 4096, 4, 8), (512, 12288, 8, 8), (64, 400, 2, 8), (32, 16, 3, 8),
    (96, 1024, 2, 32), (40, 256, 1, 2)])
def test_interleaved_rows(rows, cols, batch, R):
    """Weights compressed with R rows interleaved per 16 columns: the plain
    decode gives the interleaved order bit for bit, and the fused product
    is within the fp32 bound of the oracle's product."""
    w = _weights(rows, cols, 900 + rows + R)
    h = df11.compress(workloads.as_numpy_u16(w), interleave=R)
    assert h.interleave == R and h.shape == (rows, cols)
    d = df11.to_device(h, "cuda")
    out = df11.decode(d)
    torch.cuda.synchronize()
    want = df11.interleave_rows(workloads.as_numpy_u16(w), R)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
    x = _acts(batch, cols, rows + 7)
    y = torch.empty(batch, rows, dtype=torch.float32, device="cuda")
    err = df11.new_error_word()
    df11.decode_gemv([d], [x.cuda().view(torch.bfloat16)], [y], err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    xu = workloads.as_numpy_u16(x)
    ref = oracle.gemv(h.bitstream, h.code_lengths, h.sign_mantissa, h.n, cols, xu, interleave=R)
    W = np.abs(oracle.bf16_to_f64(workloads.as_numpy_u16(w))).reshape(rows, cols)
    g = cols * U32 / (1 - cols * U32)
    bound = g * (np.abs(oracle.bf16_to_f64(xu)).reshape(batch, cols) @ W.T)
    got = y.double().cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound), float(np.abs(got - ref).max())


def test_interleaved_build_on_device_matches_host():
    w = _weights(256, 1024, 77).cuda()
    dh = df11.to_device(df11.compress(workloads.as_numpy_u16(w.cpu()), interleave=8), "cuda")
    dd = df11.compress_on_device(w, interleave=8)
    torch.cuda.synchronize()
    assert dd.interleave == 8 and dd.shape == (256, 1024)
    for f in ("bitstream", "gaps", "chunk_counts", "sign_mantissa"):
        assert torch.equal(getattr(dd, f), getattr(dh, f)), f
