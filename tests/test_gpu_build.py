"""Device-side format builder (df11_gpu_build_begin / _finish) against the
host builder and the oracle.

Byte identity is the bar: every buffer and every parameter the device
builder writes must equal what the host builder writes for the same words
(the host builder is itself pinned to the oracle's encoder in
test_builder_vs_oracle.py), and the result must decode to the original
words.  Cases cover several pack blocks with a ragged tail, the empty and
one-element tensors, one exponent only, 8-bit codes, the multi-level tables
of the adversarial mix, 32-bit codewords, every chunk size the format
allows, and input that is not 16-byte aligned (the scalar load path).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

df11 = pytest.importorskip("huffman_decode_df11_b200")

_BUFFERS = ("bitstream", "gaps", "chunk_counts", "block_out_pos", "luts", "code_lengths",
            "sign_mantissa")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _host_bytes(h, f):
    return np.ascontiguousarray(getattr(h, f)).view(np.uint8)


def _same_as_host(bits: torch.Tensor, C=24, T=256):
    """Build on the device from `bits` (a CUDA tensor of BF16 words) and
    compare with the host builder; returns the device tensor."""
    w_np = workloads.as_numpy_u16(bits.cpu())
    h = df11.compress(w_np, C, T)
    d = df11.compress_on_device(bits, C, T)
    torch.cuda.synchronize()
    for f, _ in df11.Params._fields_:
        assert getattr(d.params, f) == getattr(h.params, f), f
    for f in _BUFFERS:
        got = getattr(d, f).cpu().numpy().view(np.uint8)
        want = _host_bytes(h, f)
        assert got.shape == want.shape, f
        assert np.array_equal(got, want), f
    assert d.shape == tuple(bits.shape)
    return d, h, w_np


def _decodes_to(d, w_np):
    err = df11.new_error_word()
    out = df11.decode(d, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), w_np)


# around the histogram's steps (2048) and the pack tiles (4096 elements, 16
# units of 256); 1,000,003 and 5,000,011 span hundreds of tiles, so that the
# look-back reads past 32 predecessors
@pytest.mark.parametrize("n", [0, 1, 2, 7, 8, 9, 255, 256, 257, 2047, 2048, 2049,
                               3 * 2048 + 77, 4095, 4096, 4097, 3 * 4096 + 1,
                               37 * 4096 + 2049, 1_000_003, 5_000_011])
def test_gaussian_sizes(n):
    bits = workloads.gaussian_bf16(n, 0.02, 500 + n, device="cuda")
    d, h, w = _same_as_host(bits)
    if n:
        _decodes_to(d, w)


@pytest.mark.parametrize("C,T", [(4, 128), (8, 256), (16, 256), (24, 256), (28, 1024),
                                 (8, 512)])
def test_chunk_and_block_sizes(C, T):
    bits = workloads.gaussian_bf16(777_777, 0.02, C * 1000 + T, device="cuda")
    d, h, w = _same_as_host(bits, C, T)
    if df11.supported(C, T):
        _decodes_to(d, w)


def test_matches_the_oracle_encoder():
    bits = workloads.adversarial_mix(1 << 18, 21, device="cuda")
    d, h, w = _same_as_host(bits, 8, 256)
    o = oracle.encode(w, 8, 256)
    assert np.array_equal(d.bitstream.cpu().numpy(), o.bitstream)
    assert np.array_equal(d.code_lengths.cpu().numpy(), o.code_lengths)


def test_adversarial_multilevel_tables():
    bits = workloads.adversarial_mix(1 << 22, 4, device="cuda")
    d, h, w = _same_as_host(bits)
    assert d.params.num_luts > 1
    _decodes_to(d, w)


def test_fibonacci_32_bit_codewords():
    bits = workloads.fibonacci_exponents(0, device="cuda")
    d, h, w = _same_as_host(bits)
    assert d.params.max_len == 32
    _decodes_to(d, w)


def test_every_bf16_pattern_and_one_exponent():
    d, h, w = _same_as_host(workloads.all_bf16_patterns(device="cuda"))
    _decodes_to(d, w)
    one = torch.full((12345,), 0x3F80, dtype=torch.int16, device="cuda")
    d, h, w = _same_as_host(one)
    assert d.params.max_len == 1
    _decodes_to(d, w)


def test_unaligned_input_takes_the_scalar_loads():
    base = workloads.gaussian_bf16(300_001, 0.02, 9, device="cuda")
    view = base[3:]  # 6 bytes past a 16-byte boundary
    assert view.data_ptr() % 16
    d, h, w = _same_as_host(view)
    _decodes_to(d, w)


def test_bf16_dtype_and_shape_kept():
    x = torch.randn(333, 517, device="cuda", dtype=torch.float32).mul_(0.02).to(torch.bfloat16)
    d = df11.compress_on_device(x)
    assert d.shape == (333, 517)
    out = df11.decode(d)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16).view(333, 517), x.view(torch.int16))


def test_argument_errors():
    x = workloads.gaussian_bf16(1000, 0.02, 1, device="cuda")
    with pytest.raises(df11.Df11Error):
        df11.compress_on_device(x, chunk_bytes=6)
    with pytest.raises(df11.Df11Error):
        df11.compress_on_device(x, threads_per_block=200)
    with pytest.raises(ValueError):
        df11.compress_on_device(x.cpu())
    with pytest.raises(TypeError):
        df11.compress_on_device(x.float())


def test_runs_of_long_codewords():
    """A thread's 8 codewords longer than 64 bits in total (a run of rare
    exponents among one common one) take the word-by-word packing path."""
    common = np.full(300_000, 240 << 7, np.uint16)
    rare = ((np.arange(2000) % 200 + 20) << 7).astype(np.uint16)
    w = np.concatenate([common[:150_001], rare, common[150_001:]])
    bits = torch.from_numpy(w.view(np.int16)).cuda()
    d, h, w = _same_as_host(bits)
    lens = h.code_lengths.astype(np.int64)[(w.astype(np.int64) >> 7) & 0xFF]
    per_thread = np.add.reduceat(lens, np.arange(0, len(lens), 8))
    assert per_thread.max() > 64  # the case this test is for
    _decodes_to(d, w)


def test_batched_builds_equal_single_builds():
    """Several tensors in one begin/finish pair (one synchronisation per
    phase): each byte-identical to the host builder, empty and unaligned
    ones included."""
    base = workloads.gaussian_bf16(300_001, 0.02, 31, device="cuda")
    bits = [workloads.gaussian_bf16(1_000_003, 0.02, 30, device="cuda"),
            torch.zeros(0, dtype=torch.int16, device="cuda"),
            base[3:],
            workloads.adversarial_mix(1 << 20, 32, device="cuda"),
            workloads.gaussian_bf16(2049, 0.5, 33, device="cuda")]
    ds = df11.compress_on_device_batched(bits, 24, 256)
    torch.cuda.synchronize()
    assert len(ds) == len(bits)
    for b, d in zip(bits, ds):
        w_np = workloads.as_numpy_u16(b.cpu())
        h = df11.compress(w_np, 24, 256)
        for f, _ in df11.Params._fields_:
            assert getattr(d.params, f) == getattr(h.params, f), f
        for f in _BUFFERS:
            assert np.array_equal(getattr(d, f).cpu().numpy().view(np.uint8), _host_bytes(h, f)), f
        if h.n:
            _decodes_to(d, w_np)


def test_many_tensors_in_one_call():
    """Forty tensors in one call, more than one histogram launch takes (32),
    with more tiles (16384 elements) than the histogram grid has blocks, so
    that blocks cross from one tensor to the next: sizes from empty to two
    million elements, some views that start off a 16-byte boundary, and
    tensors of other exponent spreads.  Each must equal the host builder's
    output byte for byte."""
    rng = np.random.default_rng(7)
    bits = []
    for i in range(40):
        kind = i % 5
        if kind == 0:
            n = int(rng.integers(0, 3))
        elif kind == 1:
            n = int(rng.integers(1, 20000))
        else:
            n = int(rng.integers(200_000, 2_000_000))
        std = float(rng.choice([0.02, 0.5, 3.0]))
        w = workloads.gaussian_bf16(n + 5, std, 100 + i, device="cuda")
        bits.append(w[5:] if i % 3 == 0 else w[:n])
    tiles = sum((b.numel() + 16383) // 16384 for b in bits)
    assert tiles > 148 * 4  # more tiles than the histogram grid's blocks
    ds = df11.compress_on_device_batched(bits, 24, 256)
    torch.cuda.synchronize()
    for b, d in zip(bits, ds):
        w_np = workloads.as_numpy_u16(b.cpu())
        h = df11.compress(w_np, 24, 256)
        for f, _ in df11.Params._fields_:
            assert getattr(d.params, f) == getattr(h.params, f), f
        for f in _BUFFERS:
            assert np.array_equal(getattr(d, f).cpu().numpy().view(np.uint8), _host_bytes(h, f)), f
    _decodes_to(ds[2], workloads.as_numpy_u16(bits[2].cpu()))


# --- randomised: skewed exponent histograms, every valid chunk size ----------

from hypothesis import given, settings, strategies as st  # noqa: E402


@st.composite
def _skewed_words(draw):
    """BF16 words whose exponents follow a random geometric histogram over a
    random subset of exponent values, random sign and mantissa bits."""
    k = draw(st.integers(1, 40))
    exps = draw(st.lists(st.integers(0, 255), min_size=k, max_size=k, unique=True))
    ratio = draw(st.sampled_from([1.0, 1.5, 2.0, 3.0]))
    n = draw(st.integers(0, 60000))
    rng = np.random.default_rng(draw(st.integers(0, 2 ** 31 - 1)))
    p = ratio ** -np.arange(k, dtype=np.float64)
    e = rng.choice(np.array(exps, dtype=np.uint32), size=n, p=p / p.sum())
    sm = rng.integers(0, 256, size=n, dtype=np.uint32)
    return (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)


@settings(max_examples=25, deadline=None)
@given(_skewed_words(), st.sampled_from([4, 8, 12, 16, 20, 24, 28]),
       st.sampled_from([128, 256, 512, 1024]))
def test_random_histograms_device_matches_host(w, C, T):
    bits = torch.from_numpy(w.view(np.int16)).cuda()
    d, h, w_np = _same_as_host(bits, C, T)
    if h.n and df11.supported(C, T):
        _decodes_to(d, w_np)


def test_tie_breaks_match_hand_worked_golden(golden_dir):
    """The device builder's code on the hand-worked tie cases
    (tests/golden/huffman_ties.json): the golden's lengths, and the host
    builder's bytes."""
    import json
    import os
    fx = json.load(open(os.path.join(golden_dir, "huffman_ties.json")))
    rng = np.random.default_rng(5)
    for case in fx["huffman"]:
        words = []
        for s, c in sorted((int(k), v) for k, v in case["weights"].items()):
            words += [((120 + s) << 7) | ((7 * i + s) & 0x7F) for i in range(c)]
        w = np.array(words, np.uint16)[rng.permutation(len(words))]
        d, h, w_np = _same_as_host(torch.from_numpy(w.view(np.int16)).cuda())
        lens = d.code_lengths.cpu().numpy()
        for s, l in case["lengths"].items():
            assert int(lens[120 + int(s)]) == l, case["weights"]
        _decodes_to(d, w_np)
