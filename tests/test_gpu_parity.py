"""CUDA decode path (libdf11.so, sm_100a) against the CPU oracle.

Bit-exact is the only bar: the decoded BF16 words must equal the oracle's
decode of the same stream element by element, and the original tensor.
Oracle-sized cases are compared in full; full-size workloads are compared
with the original tensor on the device (the round-trip property) and with the
oracle on sampled blocks, decoded one by one from their start bits.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

df11 = pytest.importorskip("huffman_decode_df11_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _decode(h, stream=None, counts=True, table=True):
    d = df11.to_device(h, "cuda", decode_table=table)
    err = df11.new_error_word()
    out = df11.decode(d, err=err, stream=stream, counts=counts)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    return out


COUNTS = pytest.mark.parametrize("counts", [True, False], ids=["counts", "no_counts"])


def _gpu_vs_oracle_full(w_np, C=8, T=256, counts=True, table=True):
    h = df11.compress(w_np, C, T)
    out = _decode(h, counts=counts, table=table).view(torch.int16).cpu().numpy().view(np.uint16)
    ref, end, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, h.n)
    assert end == h.params.total_bits
    assert np.array_equal(out, ref)       # GPU == oracle, element by element
    assert np.array_equal(out, w_np)      # == the encoded tensor
    return h


# --- oracle-sized cases, compared in full ---------------------------------

@pytest.mark.parametrize("case", ["gaussian", "adversarial", "fibonacci", "patterns", "few"])
@pytest.mark.parametrize("C", [8, 16, 24])
def test_without_decode_table(case, C):
    """Every thread block derives the decode table itself (no
    df11_build_decode_table): same output as with it."""
    if case == "gaussian":
        w = workloads.as_numpy_u16(workloads.gaussian_bf16(1_000_003, 0.02, 7))
    elif case == "adversarial":
        w = workloads.as_numpy_u16(workloads.adversarial_mix(1 << 20, 3))
    elif case == "fibonacci":
        w = workloads.as_numpy_u16(workloads.fibonacci_exponents(1, symbols=26))
    elif case == "patterns":
        w = np.random.default_rng(1).permutation(
            workloads.as_numpy_u16(workloads.all_bf16_patterns()))
    else:  # three exponents: codewords of at most 2 bits (unmasked walk)
        rng = np.random.default_rng(2)
        w = ((rng.integers(120, 123, 200_001) << 7) | rng.integers(0, 128, 200_001)).astype(np.uint16)
    _gpu_vs_oracle_full(w, C=C, table=False)
    _gpu_vs_oracle_full(w, C=C, table=True)


def test_decode_table_holds_the_rotated_format_tables():
    """The first 1280 bytes of the decode table are the code lengths indexed
    by rotated exponent and table 0 with rotated exponent bytes."""
    w = workloads.as_numpy_u16(workloads.adversarial_mix(1 << 18, 4))
    h = df11.compress(w)
    d = df11.to_device(h, "cuda")
    t = d.decode_table.cpu().numpy()
    assert t.size == df11.DF11_DECODE_TABLE_BYTES
    rot = lambda e: ((e >> 1) | ((e & 1) << 7)) & 0xFF
    lens = np.zeros(256, np.uint8)
    for e in range(256):
        lens[rot(e)] = h.code_lengths[e]
    assert np.array_equal(t[:256], lens)
    lut0 = t[256:1280].view(np.uint32)
    for i, e in enumerate(h.luts[:256]):
        e = int(e) & 0x3FFFFFFF
        if (e >> 24) & 15:
            e = (e & 0xFF000000) | rot(e & 0xFF) | (rot((e >> 8) & 0xFF) << 8) | (rot((e >> 16) & 0xFF) << 16)
        assert int(lut0[i]) == e

@COUNTS
@pytest.mark.parametrize("C,T", [(8, 256), (4, 256), (16, 256), (24, 256), (8, 128), (8, 512)])
def test_single_matrix_all_kernel_shapes(C, T, counts):
    w = workloads.as_numpy_u16(workloads.single_matrix(0))
    _gpu_vs_oracle_full(w, C, T, counts)


@COUNTS
@pytest.mark.parametrize("n", [1, 2, 7, 31, 32, 33, 255, 256, 257, 4095, 6399,
                               6400, 6401, 65537, 1_000_003])
def test_ragged_sizes(n, counts):
    w = workloads.as_numpy_u16(workloads.gaussian_bf16(n, 0.02, 100 + n))
    _gpu_vs_oracle_full(w, counts=counts)


@COUNTS
@pytest.mark.parametrize("C", [16, 24])
def test_ragged_sizes_around_warp_and_block_ranges(C, counts):
    """Prefixes of one tensor ending one element before, at and after the
    first block's and the first warp's element counts, at the wider chunks."""
    base = workloads.as_numpy_u16(workloads.gaussian_bf16(200_000, 0.02, 31))
    h = df11.compress(base, C, 256)
    block_n = int(h.block_out_pos[1])
    warp_n = int(h.chunk_counts[:32].sum())
    sizes = {1, 33, warp_n - 1, warp_n, warp_n + 1, block_n - 1, block_n, block_n + 1,
             2 * block_n + 1, 3 * block_n + warp_n}
    for n in sorted(sizes):
        _gpu_vs_oracle_full(base[:n], C=C, counts=counts)


@COUNTS
def test_every_bf16_pattern(counts):
    w = workloads.as_numpy_u16(workloads.all_bf16_patterns())
    _gpu_vs_oracle_full(w, counts=counts)
    # shuffled, so that every block holds many exponents
    rng = np.random.default_rng(0)
    _gpu_vs_oracle_full(rng.permutation(w), counts=counts)


@COUNTS
def test_single_symbol_streams(counts):
    _gpu_vs_oracle_full(np.zeros(300_001, np.uint16), counts=counts)         # +0.0 only
    _gpu_vs_oracle_full(np.full(300_001, 0x8000, np.uint16), counts=counts)  # -0.0 only
    # one exponent, random sign/mantissa: a 1-bit code, 16384 per block
    rng = np.random.default_rng(1)
    sm = rng.integers(0, 256, 500_000)
    w = (((sm & 0x80) << 8) | (120 << 7) | (sm & 0x7F)).astype(np.uint16)
    h = _gpu_vs_oracle_full(w, counts=counts)
    assert h.params.max_block_elems == 8 * 8 * 256


@COUNTS
def test_adversarial_mix_multilevel_tables(counts):
    w = workloads.as_numpy_u16(workloads.adversarial_mix(1 << 22, 4))
    h = _gpu_vs_oracle_full(w, counts=counts)
    assert h.params.num_luts > 1


@COUNTS
def test_fibonacci_32_bit_codewords(counts):
    w = workloads.as_numpy_u16(workloads.fibonacci_exponents(0))
    h = _gpu_vs_oracle_full(w, counts=counts)
    assert h.params.max_len == 32


@COUNTS
def test_few_codewords_no_masking(counts):
    # longest codeword <= 10 bits: the kernel checks region ends per lookup
    rng = np.random.default_rng(11)
    e = rng.choice(np.arange(120, 126), size=400_003, p=[.4, .25, .15, .1, .06, .04])
    sm = rng.integers(0, 256, e.size)
    w = (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
    h = _gpu_vs_oracle_full(w, counts=counts)
    assert h.params.max_len <= 10


@COUNTS
def test_many_deep_tables_read_from_global_memory(counts):
    # near-uniform exponents over a wide range with a heavy head: many
    # sub-tables, more than the kernel keeps in shared memory
    rng = np.random.default_rng(7)
    e = np.concatenate([rng.integers(0, 256, 400_000),
                        np.full(1_600_000, 126), rng.integers(110, 130, 500_000)])
    rng.shuffle(e)
    sm = rng.integers(0, 256, e.size)
    w = (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
    h = _gpu_vs_oracle_full(w, counts=counts)
    assert h.params.num_luts > 9


@COUNTS
def test_block_scaled_batched_against_oracle(counts):
    ts = workloads.block_tensors(5, scale=8)
    hs = [df11.compress(workloads.as_numpy_u16(t.bits)) for t in ts]
    ds = [df11.to_device(h) for h in hs]
    outs = [df11.empty_output(d) for d in ds]
    err = df11.new_error_word()
    df11.decode_batched(ds, outs, err=err, counts=counts)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for t, h, o in zip(ts, hs, outs):
        ref, _, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, h.n)
        got = o.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, ref)
        assert np.array_equal(got, workloads.as_numpy_u16(t.bits))


def test_batched_more_than_one_launch_and_empty_tensors():
    ws = [workloads.gaussian_bf16(n, 0.02, n) for n in
          [0, 5000, 1, 70000, 0, 123457] + [20000 + 37 * i for i in range(15)]]
    hs = [df11.compress(w) for w in ws]
    ds = [df11.to_device(h) for h in hs]
    for i, d in enumerate(ds):  # mix: every third tensor without its counts
        if i % 3 == 2:
            d.chunk_counts = None
    outs = [df11.empty_output(d) for d in ds]
    err = df11.new_error_word()
    df11.decode_batched(ds, outs, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for w, o in zip(ws, outs):
        assert torch.equal(o.view(torch.int16).cpu(), w)


def test_side_stream():
    w = workloads.single_matrix(9)
    h = df11.compress(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = _decode(h, stream=s)
    assert torch.equal(out.view(torch.int16).cpu(), w)


# --- full sizes (the benchmark's launch configuration: C=8, T=256) --------

def _sampled_blocks_vs_oracle(h, out_cpu_u16, samples=12):
    """Decode sampled blocks with the oracle from their first codeword."""
    p = h.params
    T, C = p.threads_per_block, p.chunk_bytes
    gaps = np.unpackbits(h.gaps)
    nb = p.num_blocks
    picks = sorted(set([0, nb - 1] + list(np.random.default_rng(0).integers(0, nb, samples))))
    for b in picks:
        c = b * T
        g = int("".join(str(int(x)) for x in gaps[5 * c:5 * c + 5]), 2)
        start = c * C * 8 + g
        lo, hi = int(h.block_out_pos[b]), int(h.block_out_pos[b + 1])
        if hi == lo:
            continue
        ref, _, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa[lo:],
                                  hi - lo, start_bit=start)
        assert np.array_equal(out_cpu_u16[lo:hi], ref), b


def _full_size(bits_dev: torch.Tensor, counts=True):
    h = df11.compress(bits_dev)
    d = df11.to_device(h)
    err = df11.new_error_word()
    out = df11.decode(d, err=err, counts=counts)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    assert torch.equal(out.view(torch.int16), bits_dev)   # round trip, on device
    _sampled_blocks_vs_oracle(h, out.view(torch.int16).cpu().numpy().view(np.uint16))
    return h


def test_full_block_batched():
    ts = workloads.block_tensors(0, device="cuda")
    hs = [df11.compress(t.bits) for t in ts]
    ds = [df11.to_device(h) for h in hs]
    outs = [df11.empty_output(d) for d in ds]
    err = df11.new_error_word()
    df11.decode_batched(ds, outs, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for t, h, o in zip(ts, hs, outs):
        assert torch.equal(o.view(torch.int16), t.bits)
        _sampled_blocks_vs_oracle(h, o.view(torch.int16).cpu().numpy().view(np.uint16), 4)


def test_full_adversarial_64m():
    h = _full_size(workloads.adversarial_mix(64 * 1024 * 1024, 0, device="cuda"))
    assert h.params.num_luts >= 4


@COUNTS
def test_full_embedding_622m(counts):
    _full_size(workloads.embedding(0, device="cuda"), counts)


# --- corrupted inputs: flagged, never a fault ------------------------------

def _decode_with_err(d, counts=True):
    err = df11.new_error_word()
    out = df11.decode(d, err=err, counts=counts)
    torch.cuda.synchronize()
    return out, int(err.item())


@COUNTS
def test_corrupt_block_positions_are_flagged(counts):
    w = workloads.single_matrix(1)
    h = df11.compress(w)
    d = df11.to_device(h)
    d.block_out_pos[1] += 1
    _, code = _decode_with_err(d, counts)
    assert code in (1, 5)  # COUNT or CAPACITY
    d = df11.to_device(h)
    d.block_out_pos[-1] += 1000  # past n
    _, code = _decode_with_err(d, counts)
    assert code == 5


@COUNTS
@pytest.mark.parametrize("table", [True, False], ids=["table", "no_table"])
def test_corrupt_tables_are_flagged(counts, table):
    # the decode table is derived from the format's tables: corrupt those,
    # then derive it again (or let every thread block derive it)
    w = workloads.adversarial_mix(1 << 20, 2)
    h = df11.compress(w)
    d = df11.to_device(h, decode_table=False)
    d.luts[: 256].zero_()      # every level-0 entry invalid
    if table:
        d.decode_table = df11.build_decode_table(d)
    _, code = _decode_with_err(d, counts)
    assert code == 3
    d = df11.to_device(h, decode_table=False)
    d.code_lengths.zero_()     # no codeword can be consumed on the slow path
    if table:
        d.decode_table = df11.build_decode_table(d)
    _, code = _decode_with_err(d, counts)
    assert code in (1, 2, 3)


def test_corrupt_decode_table_is_flagged():
    w = workloads.adversarial_mix(1 << 20, 5)
    h = df11.compress(w)
    d = df11.to_device(h)
    d.decode_table.zero_()     # no codeword resolves
    _, code = _decode_with_err(d, True)
    assert code == 3


def test_corrupt_chunk_counts_are_flagged():
    w = workloads.single_matrix(4)
    h = df11.compress(w)
    d = df11.to_device(h)
    d.chunk_counts[10] += 1
    d.chunk_counts[11] -= 1      # block total unchanged: caught per thread
    out, code = _decode_with_err(d)
    # the walk counted by chunk 11 stops short of its last bit (count error),
    # the one counted by chunk 10 runs past it (overrun): either comes first
    assert code in (1, 2)
    d = df11.to_device(h)
    d.chunk_counts[300] += 3     # block total changed: caught by the scan
    _, code = _decode_with_err(d)
    assert code == 1
    out = _decode(h)             # the context is still healthy
    assert torch.equal(out.view(torch.int16).cpu(), w)


@COUNTS
def test_corrupt_bitstream_never_faults(counts):
    w = workloads.single_matrix(2)
    h = df11.compress(w)
    rng = np.random.default_rng(3)
    for trial in range(8):
        d = df11.to_device(h)
        idx = torch.as_tensor(rng.integers(0, h.bitstream.size - 16, 50), device="cuda")
        d.bitstream[idx] ^= torch.as_tensor(rng.integers(1, 256, 50), dtype=torch.uint8,
                                            device="cuda")
        # Huffman streams carry no checksum: a flip is flagged or decodes to
        # other values; either way the call completes inside its buffers
        _, code = _decode_with_err(d, counts)
        assert code in (0, 1, 2, 3)
    out = _decode(h)
    assert torch.equal(out.view(torch.int16).cpu(), w)  # context still healthy


def test_host_side_argument_errors():
    h = df11.compress(workloads.single_matrix(0))
    d = df11.to_device(h)
    out = df11.empty_output(d)
    with pytest.raises(df11.Df11Error, match="ALIGN"):
        big = torch.empty(d.n + 1, dtype=torch.bfloat16, device="cuda")
        df11.decode(d, out=big[1:])
    with pytest.raises(ValueError):
        df11.decode(d, out=out[:-1])


def test_tensors_loaded_from_a_file_decode_bit_exact(tmp_path):
    from huffman_decode_df11_b200 import serialization as ser
    ws = {"a": workloads.as_numpy_u16(workloads.adversarial_mix(1 << 20, 11)),
          "b": workloads.as_numpy_u16(workloads.gaussian_bf16(777_777, 0.02, 12))}
    path = str(tmp_path / "w.df11")
    ser.save(path, {k: df11.compress(v) for k, v in ws.items()})
    for k, h in ser.load(path).items():
        out = _decode(h).view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(out, ws[k])


def test_offload_pipeline_decodes_every_layer_bit_exact():
    """Layers packed in pinned host memory, copied and decoded through two
    device slots; every layer's output checked right after its decode, and
    a second run of the same pipeline."""
    from huffman_decode_df11_b200 import offload
    rng = np.random.default_rng(5)
    layers = []
    for i in range(5):  # sizes differ, so the slots are reused at several offsets
        ws = [workloads.as_numpy_u16(workloads.gaussian_bf16(int(rng.integers(1, 400_000)),
                                                             0.02, 20 + 3 * i + j))
              for j in range(3)]
        if i == 2:
            ws.append(workloads.as_numpy_u16(workloads.adversarial_mix(1 << 18, 7)))
        layers.append(ws)
    packed = [offload.pack_layer([df11.compress(w) for w in ws]) for ws in layers]
    # one scratch buffer for every layer; outputs start 16-byte aligned
    scratch = torch.empty(max(sum(len(w) + 8 for w in ws) for ws in layers),
                          dtype=torch.int16, device="cuda")
    outs = []
    for ws in layers:
        off, o = 0, []
        for w in ws:
            o.append(scratch[off:off + len(w)])
            off = (off + len(w) + 7) // 8 * 8
        outs.append(o)
    pipe = offload.OffloadPipeline(packed, outs)
    err = df11.new_error_word()
    got = {}

    def check(i):  # copies the layer's output before the next decode overwrites it
        got[i] = [o.clone() for o in outs[i]]

    for _ in range(2):
        got.clear()
        pipe.run(err=err, after_layer=check)
        torch.cuda.synchronize()
        df11.check_device_error(err)
        for i, ws in enumerate(layers):
            for o, w in zip(got[i], ws):
                assert np.array_equal(o.cpu().numpy().view(np.uint16), w)
    assert pipe.h2d_bytes == sum(p.nbytes for p in packed)
