"""Fused decode and matrix product on the tensor cores (df11_decode_gemm)
against the oracle.

Weights are compressed with 128 rows interleaved per 16 columns, so that the
stream holds 128 x 16 tiles; the kernel decodes them into shared memory and
multiplies them by the activations with tcgen05.mma (BF16 operands, fp32
accumulation in tensor memory), then adds each 128-row block's sums to y
with fp32 atomics.  The oracle decodes the stream bit by bit, reads the
interleaved order back by index and multiplies in float64 (oracle.gemv).
Every product of two BF16 values is exact in fp32; only the sums round, so
each output is held to gamma_K * sum |w x| of the exact value (K = cols,
the bound for a sum of K terms in any order; with y += one more term).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

df11 = pytest.importorskip("huffman_decode_df11_b200")

U32 = 2.0 ** -24
R = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _gamma(k):
    return k * U32 / (1 - k * U32)


def _weights(rows, cols, seed, std=None):
    std = std if std is not None else 1.0 / np.sqrt(cols)
    return workloads.gaussian_bf16(rows * cols, std, seed).view(rows, cols)


def _acts(batch, cols, seed):
    return workloads.gaussian_bf16(batch * cols, 1.0, 10_000 + seed).view(batch, cols)


def _compressed(w, C=8):
    rows, cols = w.shape
    h = df11.compress(workloads.as_numpy_u16(w).reshape(rows, cols), C, 256, interleave=R)
    return h, df11.to_device(h, "cuda")


def _check(h, w, x, y_gpu, y0=None):
    """y_gpu against the oracle's float64 product of the decoded stream."""
    rows, cols = w.shape
    xu = workloads.as_numpy_u16(x)
    ref = oracle.gemv(h.bitstream, h.code_lengths, h.sign_mantissa, h.n, cols, xu,
                      interleave=R)
    W = np.abs(oracle.bf16_to_f64(workloads.as_numpy_u16(w))).reshape(rows, cols)
    X = np.abs(oracle.bf16_to_f64(xu)).reshape(-1, cols)
    mag = X @ W.T
    if y0 is None:
        bound = _gamma(cols) * mag
    else:
        ref = ref + y0
        bound = _gamma(cols + 1) * (mag + np.abs(y0))
    got = y_gpu.double().cpu().numpy().reshape(ref.shape)
    err = np.abs(got - ref)
    assert np.all(err <= bound), (float(err.max()), float(bound[err > bound].min()))


@pytest.mark.parametrize("rows,cols,batch,C", [
    (128, 16, 16, 8),        # one tile
    (256, 512, 8, 8),        # two row blocks, one unit each; batch padded to 16
    (384, 1040, 16, 8),      # 65 column groups: a short last unit
    (1024, 4096, 1, 8),
    (1024, 4096, 17, 8),     # batch 17: N = 32, rows 17-31 of the tile zero
    (1024, 4096, 64, 8),
    (512, 4096, 128, 8),
    (1024, 4096, 32, 16),
    (1024, 12288, 48, 8)])
def test_gemm_within_fp32_bound(rows, cols, batch, C):
    w = _weights(rows, cols, rows * 7 + cols + batch)
    h, d = _compressed(w, C)
    x = _acts(batch, cols, rows + cols)
    y = torch.full((batch, rows), 123.0, dtype=torch.float32, device="cuda")
    err = df11.new_error_word()
    df11.decode_gemm([d], [x.cuda().view(torch.bfloat16)], [y], err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    _check(h, w, x, y)


def test_gemm_accumulates_and_takes_several_weights():
    shapes = [(256, 4096), (1024, 4096), (128, 1024), (640, 2048)]
    batch = 24
    ws = [_weights(r, c, 31 + i) for i, (r, c) in enumerate(shapes)]
    hs, ds = zip(*[_compressed(w) for w in ws])
    xs = [_acts(batch, c, 40 + i) for i, (_, c) in enumerate(shapes)]
    y0s = [np.random.default_rng(i).standard_normal((batch, r)).astype(np.float32)
           for i, (r, _) in enumerate(shapes)]
    ys = [torch.from_numpy(y0).cuda() for y0 in y0s]
    err = df11.new_error_word()
    df11.decode_gemm(list(ds), [x.cuda().view(torch.bfloat16) for x in xs], ys,
                     accumulate=True, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for h, w, x, y, y0 in zip(hs, ws, xs, ys, y0s):
        _check(h, w, x, y, y0.astype(np.float64))


def test_gemm_strided_activations_and_outputs():
    rows, cols, batch = 512, 2048, 20
    w = _weights(rows, cols, 77)
    h, d = _compressed(w)
    x = _acts(batch, cols, 78)
    xbig = torch.zeros(batch, cols + 64, dtype=torch.int16, device="cuda")
    xbig[:, :cols] = x.cuda()
    ybig = torch.full((batch, rows + 32), 7.0, dtype=torch.float32, device="cuda")
    err = df11.new_error_word()
    df11.decode_gemm([d], [xbig[:, :cols].view(torch.bfloat16)], [ybig[:, :rows]], err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    _check(h, w, x, ybig[:, :rows].contiguous())
    assert torch.all(ybig[:, rows:] == 7.0)  # nothing written past the rows


def test_gemm_matches_decode_then_matmul():
    """The same product as decoding (plain decode, interleaved order read
    back) and multiplying in float64 on the device."""
    rows, cols, batch = 2048, 4096, 64
    w = _weights(rows, cols, 90)
    h, d = _compressed(w)
    out = df11.decode(d)
    flat = out.view(torch.int16)
    W = df11.deinterleave_rows(flat, (rows, cols), R)
    assert torch.equal(W.cpu(), w)
    x = _acts(batch, cols, 91).cuda()
    y = torch.empty(batch, rows, dtype=torch.float32, device="cuda")
    df11.decode_gemm([d], [x.view(torch.bfloat16)], [y])
    ref = x.view(torch.bfloat16).double() @ W.view(torch.bfloat16).double().T
    mag = x.view(torch.bfloat16).double().abs() @ W.view(torch.bfloat16).double().abs().T
    assert torch.all((y.double() - ref).abs() <= _gamma(cols) * mag)


def test_gemm_argument_errors():
    w = _weights(256, 512, 5)
    h, d = _compressed(w)
    x = _acts(8, 512, 5).cuda().view(torch.bfloat16)
    y = torch.empty(8, 256, dtype=torch.float32, device="cuda")
    h_rm = df11.compress(workloads.as_numpy_u16(w), 8, 256)
    h_rm.shape = (256, 512)
    d_rm = df11.to_device(h_rm)
    with pytest.raises(ValueError):
        df11.decode_gemm([d_rm], [x], [y])  # row-major weights
    with pytest.raises(df11.Df11Error):
        df11.decode_gemm([d], [_acts(129, 512, 6).cuda().view(torch.bfloat16)],
                         [torch.empty(129, 256, device="cuda")])  # batch over 128
    h24, d24 = _compressed(w, C=24)
    with pytest.raises(df11.Df11Error, match="UNSUPPORTED"):
        df11.decode_gemm([d24], [x], [y])


def test_gemm_flags_corrupt_tables_and_stays_usable():
    w = _weights(512, 2048, 8)
    h, d = _compressed(w)
    x = _acts(16, 2048, 9).cuda().view(torch.bfloat16)
    y = torch.empty(16, 512, dtype=torch.float32, device="cuda")
    bad = df11.to_device(h, decode_table=False)
    bad.luts[:256].zero_()
    bad.decode_table = df11.build_decode_table(bad)
    err = df11.new_error_word()
    df11.decode_gemm([bad], [x], [y], err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 3  # DF11_DEV_ERR_TABLE
    err.zero_()
    df11.decode_gemm([d], [x], [y], err=err)  # the context still works
    torch.cuda.synchronize()
    df11.check_device_error(err)
    _check(h, w, x.view(torch.int16).cpu(), y)


def test_gemm_block_shapes_full_size_in_one_call():
    """The bench's launch: the seven weights of a Qwen3-8B-shaped block
    (192,937,984 elements), compressed on the device at C = 8 with 128 rows
    interleaved, times 32 activation rows, in one call; every output within
    the fp32 sum bound of the float64 product of the original weights (the
    decode is lossless, so the original weights are the exact reference;
    computed on the device, one weight at a time)."""
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (12288, 4096),
              (12288, 4096), (4096, 12288)]
    batch = 32
    ws = [workloads.gaussian_bf16(r * c, 1.0 / np.sqrt(c), 700 + i, device="cuda").view(r, c)
          for i, (r, c) in enumerate(shapes)]
    ds = df11.compress_on_device_batched(ws, 8, 256, decode_table=True, interleave=R)
    xs = [workloads.gaussian_bf16(batch * c, 1.0, 800 + i, device="cuda").view(batch, c)
          for i, (_, c) in enumerate(shapes)]
    ys = [torch.full((batch, r), 5.0, dtype=torch.float32, device="cuda") for r, _ in shapes]
    err = df11.new_error_word()
    df11.decode_gemm(ds, [x.view(torch.bfloat16) for x in xs], ys, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for w, x, y, (r, c) in zip(ws, xs, ys, shapes):
        W = w.view(torch.bfloat16).double()
        X = x.view(torch.bfloat16).double()
        ref = X @ W.T
        bound = _gamma(c) * (X.abs() @ W.abs().T)
        assert bool(torch.all((y.double() - ref).abs() <= bound)), (r, c)
        del W, X, ref, bound
