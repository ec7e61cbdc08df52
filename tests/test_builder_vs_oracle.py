"""The host format builder (libdf11.so, C++) against the oracle (plain C):
byte-identical output on every workload.  The two share no code; both follow
the same tie-break rules, so their streams, tables and metadata must agree
exactly, and the oracle's bit-serial decoder must read the builder's stream
back to the original tensor."""
import numpy as np
import pytest

import huffman_decode_df11_b200 as df11
import oracle
import workloads


def _compare(w, C, T, threads=4):
    h = df11.compress(w, C, T, threads=threads)
    f = oracle.encode(w, C, T)
    p = h.params
    assert p.n == f.n
    assert p.total_bits == f.total_bits
    assert p.num_blocks == f.num_blocks
    assert p.num_luts == f.num_luts
    assert p.max_block_elems == f.max_block_elems
    assert p.max_len == f.max_len
    assert p.max_chunk_elems == f.max_chunk_elems
    assert p.max_warp_elems == f.max_warp_elems
    assert np.array_equal(h.code_lengths, f.code_lengths)
    assert np.array_equal(h.bitstream, f.bitstream)
    assert np.array_equal(h.gaps, f.gaps_packed)
    assert np.array_equal(h.block_out_pos, f.block_out_pos)
    assert np.array_equal(h.luts, f.luts)
    assert np.array_equal(h.sign_mantissa, f.sign_mantissa)
    assert np.array_equal(h.chunk_counts, f.chunk_counts)
    return h


@pytest.mark.parametrize("C,T", [(8, 256), (4, 256), (16, 256), (24, 256), (28, 256),
                                 (8, 128), (8, 512), (24, 1024)])
def test_single_matrix(C, T):
    w = workloads.as_numpy_u16(workloads.single_matrix(0))
    _compare(w, C, T)


def test_block_tensors_scaled():
    for t in workloads.block_tensors(0, scale=16):
        _compare(workloads.as_numpy_u16(t.bits), 8, 256)


def test_adversarial_and_long_codes():
    w = workloads.as_numpy_u16(workloads.adversarial_mix(1 << 21, 1))
    h = _compare(w, 8, 256)
    assert h.params.num_luts > 1


def test_fibonacci_forces_package_merge():
    w = workloads.as_numpy_u16(workloads.fibonacci_exponents(0))
    h = _compare(w, 8, 256, threads=8)
    assert h.params.max_len == 32


@pytest.mark.parametrize("n", [0, 1, 2, 31, 32, 33, 6399, 6400, 6401, 100003])
def test_ragged_sizes(n):
    w = workloads.as_numpy_u16(workloads.gaussian_bf16(n, 0.02, 7 + n))
    _compare(w, 8, 256)


def test_special_values():
    _compare(workloads.as_numpy_u16(workloads.all_bf16_patterns()), 8, 256)
    _compare(np.zeros(70000, np.uint16), 8, 256)            # one symbol
    _compare(np.full(70000, 0x8000, np.uint16), 4, 128)     # -0.0 only


@pytest.mark.parametrize("threads", [1, 3, 8, 64])
def test_thread_count_does_not_change_the_output(threads):
    w = workloads.as_numpy_u16(workloads.adversarial_mix(300_000, 9))
    _compare(w, 8, 256, threads=threads)


def test_oracle_decodes_builder_stream():
    w = workloads.as_numpy_u16(workloads.block_tensors(3, scale=64)[4].bits)
    h = df11.compress(w, 8, 256)
    out, end, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, h.n)
    assert end == h.params.total_bits
    assert np.array_equal(out, w)


def test_builder_rejects_bad_parameters():
    w = np.zeros(10, np.uint16)
    for C, T in [(3, 256), (6, 256), (8, 100), (8, 2048), (0, 256), (32, 256), (68, 256)]:
        with pytest.raises(df11.Df11Error):
            df11.compress(w, C, T)


# --- randomised: skewed exponent histograms, every valid chunk size ----------

from hypothesis import given, settings, strategies as st  # noqa: E402


@st.composite
def _skewed_words(draw):
    """BF16 words whose exponents follow a random skewed histogram over a
    random subset of the 256 values (geometric weights give long codes),
    with random sign and mantissa bits, in random order."""
    k = draw(st.integers(1, 40))
    exps = draw(st.lists(st.integers(0, 255), min_size=k, max_size=k, unique=True))
    ratio = draw(st.sampled_from([1.0, 1.5, 2.0, 3.0]))
    n = draw(st.integers(0, 30000))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    p = ratio ** -np.arange(k, dtype=np.float64)
    e = rng.choice(np.array(exps, dtype=np.uint32), size=n, p=p / p.sum())
    sm = rng.integers(0, 256, size=n, dtype=np.uint32)
    return (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)


@settings(max_examples=60, deadline=None)
@given(_skewed_words(), st.sampled_from([4, 8, 12, 16, 20, 24, 28]),
       st.sampled_from([128, 256, 512, 1024]))
def test_random_histograms_every_chunk_size(w, C, T):
    h = _compare(w, C, T)
    if h.n:
        out, end, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, h.n)
        assert end == h.params.total_bits
        assert np.array_equal(out, w)


def _tensor_with_exponent_counts(weights, base=120):
    """BF16 words whose exponent histogram is `weights` (symbol s -> exponent
    base + s), sign and mantissa varied, in a fixed shuffled order."""
    words = []
    for s, c in sorted((int(k), v) for k, v in weights.items()):
        words += [((base + s) << 7) | ((7 * i + s) & 0x7F) | ((i & 1) << 15) for i in range(c)]
    rng = np.random.default_rng(5)
    return np.array(words, np.uint16)[rng.permutation(len(words))]


def test_tie_breaks_match_hand_worked_golden(golden_dir):
    """The host builder's Huffman tie order on the hand-worked golden cases
    (tests/golden/huffman_ties.json): code lengths and the bytes of the
    stream equal the golden's and the oracle's."""
    import json
    import os
    fx = json.load(open(os.path.join(golden_dir, "huffman_ties.json")))
    for case in fx["huffman"]:
        w = _tensor_with_exponent_counts(case["weights"])
        h = _compare(w, 8, 256)
        for s, l in case["lengths"].items():
            assert int(h.code_lengths[120 + int(s)]) == l, case["weights"]
        assert int((h.code_lengths > 0).sum()) == len(case["lengths"])
