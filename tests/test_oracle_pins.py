"""Pins of the CPU oracle to facts the pages and the mathematics fix.

Nothing here compares the oracle with itself: each test checks it against a
hand-worked fixture (tests/golden/), a brute-force search, an independent
decoding method, or a bound that any correct Huffman code obeys.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
import workloads


def _hex(s):
    return int(s, 16)


# -------------------------------------------------------------------------
# BF16 field split ("DFloat11无损压缩技术" §2.1, §2.2 item 2)

def test_field_split_matches_hand_worked_words(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "bf16_fields.json")))
    words = np.array([_hex(c["word"]) for c in fx["cases"]], np.uint16)
    exps, sm = oracle.split(words)
    for c, e, s in zip(fx["cases"], exps, sm):
        assert e == c["exponent"], c
        assert s == _hex(c["sm"]), c
        assert (s >> 7) == c["sign"] and (s & 0x7F) == c["mantissa"], c


def test_every_bf16_pattern_round_trips():
    w = workloads.as_numpy_u16(workloads.all_bf16_patterns())
    f, out = oracle.roundtrip(w, chunk_bytes=8, threads_per_block=256)
    assert np.array_equal(out, w)
    assert (f.code_lengths > 0).sum() == 256  # every exponent 0..255 occurs


# -------------------------------------------------------------------------
# Huffman code lengths: optimality by brute force, Kraft, entropy bound

def _brute_force_optimum(weights, max_len):
    """Minimum sum(w*l) over all length vectors obeying Kraft's inequality."""
    m = len(weights)
    best = None
    top = min(max_len, m - 1)
    for lens in itertools.product(range(1, top + 1), repeat=m):
        if sum(2.0 ** -l for l in lens) <= 1.0 + 1e-12:
            cost = sum(w * l for w, l in zip(weights, lens))
            if best is None or cost < best:
                best = cost
    return best


@pytest.mark.parametrize("seed", range(40))
def test_huffman_is_optimal_on_small_alphabets(seed):
    rng = np.random.default_rng(seed)
    m = int(rng.integers(2, 7))
    weights = [int(x) for x in rng.integers(1, 50, size=m)]
    hist = np.zeros(256, np.uint64)
    syms = rng.choice(256, size=m, replace=False)
    hist[syms] = weights
    lens, longest = oracle.huffman_lengths(hist)
    cost = int(sum(int(hist[s]) * int(lens[s]) for s in syms))
    assert cost == _brute_force_optimum(weights, m - 1)
    assert longest == max(int(lens[s]) for s in syms)
    assert all(lens[s] == 0 for s in range(256) if s not in set(syms.tolist()))


@pytest.mark.parametrize("seed", range(40))
@pytest.mark.parametrize("limit", [2, 3, 4])
def test_package_merge_is_optimal_under_a_length_limit(seed, limit):
    rng = np.random.default_rng(1000 + seed)
    m = int(rng.integers(2, min(7, 2 ** limit + 1)))
    # skewed weights so that the limit binds often
    weights = [int(x) for x in (2 ** rng.integers(0, 9, size=m))]
    hist = np.zeros(256, np.uint64)
    syms = rng.choice(256, size=m, replace=False)
    hist[syms] = weights
    lens, longest = oracle.package_merge_lengths(hist, limit)
    assert 1 <= longest <= limit
    kraft = sum(2.0 ** -int(lens[s]) for s in syms)
    assert kraft <= 1.0
    cost = sum(int(hist[s]) * int(lens[s]) for s in syms)
    assert cost == _brute_force_optimum(weights, limit)


def _kraft_sum_2_32(lens):
    return sum(1 << (32 - int(l)) for l in lens if l > 0)


def _entropy(hist):
    p = hist[hist > 0].astype(np.float64) / hist.sum()
    return float(-(p * np.log2(p)).sum())


def _workload_hists():
    out = {}
    w = workloads.as_numpy_u16(workloads.single_matrix(0))
    out["single_matrix"] = oracle.histogram(oracle.split(w)[0])
    for t in workloads.block_tensors(0, scale=16):
        w = workloads.as_numpy_u16(t.bits)
        out["block." + t.name] = oracle.histogram(oracle.split(w)[0])
    w = workloads.as_numpy_u16(workloads.adversarial_mix(1 << 22, 0))
    out["adversarial_4M"] = oracle.histogram(oracle.split(w)[0])
    w = workloads.as_numpy_u16(workloads.fibonacci_exponents(0))
    out["fibonacci34"] = oracle.histogram(oracle.split(w)[0])
    w = workloads.as_numpy_u16(workloads.all_bf16_patterns())
    out["all_patterns"] = oracle.histogram(oracle.split(w)[0])
    return out


@pytest.fixture(scope="module")
def workload_hists():
    return _workload_hists()


def test_kraft_equality_and_entropy_bound(workload_hists):
    for name, hist in workload_hists.items():
        lens, longest = oracle.code_lengths(hist)
        assert 1 <= longest <= 32, name
        # a complete prefix code: sum 2^-len == 1 exactly
        assert _kraft_sum_2_32(lens) == 1 << 32, name
        avg = float((hist.astype(np.float64) * lens).sum() / hist.sum())
        H = _entropy(hist)
        if name != "fibonacci34":
            assert H <= avg < H + 1, (name, H, avg)
        else:  # the length limit may cost a little, never below entropy
            assert H <= avg < H + 1.01, (name, H, avg)


def test_package_merge_equals_huffman_when_the_limit_is_slack(workload_hists):
    for name, hist in workload_hists.items():
        h_lens, h_long = oracle.huffman_lengths(hist)
        if h_long > 32:
            continue
        p_lens, p_long = oracle.package_merge_lengths(hist, 32)
        h_cost = int((hist * h_lens.astype(np.uint64)).sum())
        p_cost = int((hist * p_lens.astype(np.uint64)).sum())
        assert h_cost == p_cost, name  # two algorithms, one optimum


def test_fibonacci_weights_force_the_32_bit_cap(workload_hists):
    hist = workload_hists["fibonacci34"]
    assert int(hist.sum()) == 14_930_351  # F36 - 1
    h_lens, h_long = oracle.huffman_lengths(hist)
    assert h_long == 33
    lens, longest = oracle.code_lengths(hist)
    assert longest == 32
    assert _kraft_sum_2_32(lens) == 1 << 32
    # Bounds on the optimum of the capped problem.  Below: no code beats the
    # unconstrained Huffman optimum.  Above: an explicit 32-deep code costs one
    # bit more -- the depth-30 subtree holding F4 (depth 31), F3 (32), F1 and
    # F2 (33) becomes four leaves at depth 32: +1*3 for F4, -1*1 twice.
    p_cost = int((hist * lens.astype(np.uint64)).sum())
    h_cost = int((hist * h_lens.astype(np.uint64)).sum())
    assert h_cost <= p_cost <= h_cost + 1


def test_single_symbol_gets_one_bit():
    hist = np.zeros(256, np.uint64)
    hist[17] = 1000
    lens, longest = oracle.code_lengths(hist)
    assert longest == 1 and lens[17] == 1 and lens.sum() == 1


# -------------------------------------------------------------------------
# Canonical codes (RFC 1951 §3.2.2 worked example; prefix property)

def test_canonical_codes_match_rfc1951_example(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "canonical_rfc1951.json")))
    codes = oracle.canonical_codes(fx["lengths"])
    for s, (l, want) in enumerate(zip(fx["lengths"], fx["codes"])):
        assert format(int(codes[s]), f"0{l}b") == want


def test_canonical_codes_are_prefix_free(workload_hists):
    for name, hist in workload_hists.items():
        lens, _ = oracle.code_lengths(hist)
        codes = oracle.canonical_codes(lens)
        words = [format(int(codes[s]), f"0{int(lens[s])}b")
                 for s in range(256) if lens[s] > 0]
        assert len(set(words)) == len(words), name
        for a in words:
            for b in words:
                if a != b:
                    assert not b.startswith(a), (name, a, b)


# -------------------------------------------------------------------------
# Tie-breaks of the code construction (hand-worked cases, tests/golden/
# huffman_ties.json).  The pages are silent on ties; the format fixes them,
# so that the encoded bytes are unique.

def _ties(golden_dir):
    return json.load(open(os.path.join(golden_dir, "huffman_ties.json")))


def _hist_of(weights):
    h = np.zeros(256, np.uint64)
    for s, w in weights.items():
        h[int(s)] = w
    return h


def test_huffman_ties_match_hand_worked_golden(golden_dir):
    for case in _ties(golden_dir)["huffman"]:
        h = _hist_of(case["weights"])
        lens, longest = oracle.huffman_lengths(h)
        want = {int(s): l for s, l in case["lengths"].items()}
        assert {s: int(lens[s]) for s in want} == want, case["weights"]
        assert int(lens.sum()) == sum(want.values())  # no other symbol coded
        assert longest == max(want.values())
        assert sum(int(h[s]) * l for s, l in want.items()) == case["cost_bits"]
        # below the 32-bit cap the full construction is plain Huffman
        full, _ = oracle.code_lengths(h)
        assert np.array_equal(full, lens)
        codes = oracle.canonical_codes(lens)
        for s, bits in case["canonical"].items():
            assert format(int(codes[int(s)]), f"0{want[int(s)]}b") == bits


def test_package_merge_ties_match_hand_worked_golden(golden_dir):
    for case in _ties(golden_dir)["package_merge"]:
        h = _hist_of(case["weights"])
        lens, longest = oracle.package_merge_lengths(h, case["max_len"])
        want = {int(s): l for s, l in case["lengths"].items()}
        assert {s: int(lens[s]) for s in want} == want, case["weights"]
        assert int(lens.sum()) == sum(want.values())
        assert sum(int(h[s]) * l for s, l in want.items()) == case["cost_bits"]


def _huffman_by_rule(weights, key):
    """Textbook Huffman in plain Python with a pluggable tie order (node =
    (weight, smallest symbol, creation index, symbols)); only used to show
    that the golden cases tell tie rules apart."""
    nodes = [(w, s, i, [s]) for i, (s, w) in enumerate(sorted(weights.items()))]
    depth = {s: 0 for s in weights}
    made = len(nodes)
    while len(nodes) > 1:
        nodes.sort(key=key)
        a, b = nodes[0], nodes[1]
        for s in a[3] + b[3]:
            depth[s] += 1
        nodes = nodes[2:] + [(a[0] + b[0], min(a[1], b[1]), made, a[3] + b[3])]
        made += 1
    return depth


def test_golden_ties_tell_tie_rules_apart(golden_dir):
    """Each other plausible tie order fails at least one golden case, so a
    swapped order in the oracle (or a builder) cannot pass the pins."""
    cases = _ties(golden_dir)["huffman"]
    rules = {"larger smallest-symbol first": lambda n: (n[0], -n[1]),
             "newest node first": lambda n: (n[0], -n[2]),
             "oldest node first": lambda n: (n[0], n[2])}
    for name, key in rules.items():
        differs = False
        for case in cases:
            w = {int(s): v for s, v in case["weights"].items()}
            want = {int(s): l for s, l in case["lengths"].items()}
            got = _huffman_by_rule(w, key)
            assert sum(w[s] * got[s] for s in w) == case["cost_bits"]  # still optimal
            differs |= got != want
        assert differs, name
    # the stated rule itself reproduces every case
    for case in cases:
        w = {int(s): v for s, v in case["weights"].items()}
        assert _huffman_by_rule(w, lambda n: (n[0], n[1])) == \
            {int(s): l for s, l in case["lengths"].items()}


# -------------------------------------------------------------------------
# Hand-written bitstreams

def _golden_streams(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "bitstreams.json")))
    lens = np.zeros(256, np.uint8)
    for k, v in fx["codebook"]["lengths"].items():
        lens[int(k)] = v
    return fx, lens


def test_hand_written_streams_decode(golden_dir):
    fx, lens = _golden_streams(golden_dir)
    for st in fx["streams"]:
        bits = st["bits"]
        assert len(bits) == st["total_bits"]
        raw = np.array([_hex(b) for b in st["bytes"]] + [0] * 16, np.uint8)
        # the hex bytes are the bit string, MSB first
        unpacked = "".join(format(int(b), "08b") for b in raw)
        assert unpacked.startswith(bits)
        sm = np.array([_hex(s) for s in st["sign_mantissa"]], np.uint8)
        n = len(st["exponents"])
        out, end, starts = oracle.decode(raw, lens, sm, n, want_starts=True)
        assert end == st["total_bits"]
        assert starts.tolist() == st["starts"]
        if "words" in st:
            assert [int(x) for x in out] == [_hex(x) for x in st["words"]]
        assert [(int(x) >> 7) & 0xFF for x in out] == st["exponents"]


def test_hand_written_stream_metadata(golden_dir):
    fx, _ = _golden_streams(golden_dir)
    for st in fx["streams"]:
        C, T = st["chunk_bytes"], st["threads_per_block"]
        nb = math.ceil(st["total_bits"] / (8 * C * T))
        gaps, pos = oracle.metadata_from_starts(
            np.array(st["starts"], np.uint64), len(st["starts"]),
            st["total_bits"], C, T, nb)
        want = np.zeros(nb * T, np.uint8)
        for k, v in st["gaps_nonzero"].items():
            want[int(k)] = v
        assert np.array_equal(gaps, want)
        assert pos.tolist() == st["block_out_pos"]


def test_hand_written_stream_encodes(golden_dir):
    fx, lens = _golden_streams(golden_dir)
    for st in fx["streams"]:
        if not st["histogram_gives_codebook"]:
            continue
        sm = [_hex(s) for s in st["sign_mantissa"]]
        words = np.array([((s >> 7) << 15) | (e << 7) | (s & 0x7F)
                          for e, s in zip(st["exponents"], sm)], np.uint16)
        assert words.tolist() == [_hex(x) for x in st["words"]]
        f = oracle.encode(words, st["chunk_bytes"], st["threads_per_block"])
        assert np.array_equal(f.code_lengths, lens)
        want = [_hex(b) for b in st["bytes"]]
        assert f.bitstream[: len(want)].tolist() == want
        assert not f.bitstream[len(want):].any()
        assert f.total_bits == st["total_bits"]
        assert f.block_out_pos.tolist() == st["block_out_pos"]


# -------------------------------------------------------------------------
# Lookup tables: an independent table-walking decoder must agree with the
# bit-serial decoder on real streams.

def _read32(stream_bits: np.ndarray, pos: int) -> int:
    chunk = stream_bits[pos:pos + 32]
    v = 0
    for b in chunk:
        v = (v << 1) | int(b)
    return v << (32 - len(chunk))


def _table_walk_decode(f: oracle.OracleFormat, count: int):
    bits = np.unpackbits(f.bitstream)
    luts = f.luts
    out, pos = [], 0
    while len(out) < count:
        win = _read32(bits, pos)
        e = int(luts[win >> 24])
        nbits, nsym = (e >> 24) & 15, (e >> 28) & 3
        if nbits:
            assert nsym >= 1
            for k in range(nsym):
                if len(out) < count:
                    out.append((e >> (8 * k)) & 0xFF)
            pos += nbits
            continue
        table, level = e & 0xFFFFFF, 1
        assert table > 0, "invalid entry reached"
        while True:
            e = int(luts[table * 256 + ((win >> (24 - 8 * level)) & 0xFF)])
            if (e >> 28) & 3:
                sym = e & 0xFF
                out.append(sym)
                pos += int(f.code_lengths[sym])
                break
            table = e & 0xFFFFFF
            assert table > 0 and level < 3, "invalid entry reached"
            level += 1
    return out


@pytest.mark.parametrize("case", ["single_matrix", "adversarial", "fibonacci",
                                  "all_patterns"])
def test_lookup_tables_decode_like_the_bit_serial_decoder(case):
    if case == "single_matrix":
        w = workloads.as_numpy_u16(workloads.single_matrix(3))[:20000]
    elif case == "adversarial":
        w = workloads.as_numpy_u16(workloads.adversarial_mix(1 << 16, 2))
    elif case == "fibonacci":
        w = workloads.as_numpy_u16(workloads.fibonacci_exponents(1))[:20000]
    else:
        w = workloads.as_numpy_u16(workloads.all_bf16_patterns())
    # build the code from the whole tensor so that long codewords exist,
    # then walk the tables over a prefix of the stream
    f = oracle.encode(w, 8, 256)
    count = min(f.n, 12000)
    walked = _table_walk_decode(f, count)
    exps = oracle.split(w)[0][:count]
    assert walked == exps.tolist()
    if case in ("adversarial", "fibonacci"):
        assert f.num_luts > 1  # sub-tables were exercised
    if case == "all_patterns":  # 256 equally likely exponents: all 8 bits
        assert (f.code_lengths == 8).all() and f.num_luts == 1


def test_level0_table_of_a_complete_code_has_no_invalid_entry(workload_hists):
    for name, hist in workload_hists.items():
        lens, _ = oracle.code_lengths(hist)
        luts = oracle.build_luts(lens)
        assert (luts[:256] != 0).all(), name


# -------------------------------------------------------------------------
# Chunk gaps / block output positions: brute force on the definitions, and
# every chunk's gap really is a codeword boundary (decoding from there gives
# the right elements).

@pytest.mark.parametrize("C,T", [(4, 128), (8, 128), (8, 256), (16, 128)])
def test_gaps_and_block_positions_brute_force(C, T):
    w = workloads.as_numpy_u16(workloads.adversarial_mix(30000, 5))
    f = oracle.encode(w, C, T)
    _, end, starts = oracle.decode(f.bitstream, f.code_lengths,
                                   f.sign_mantissa, f.n, want_starts=True)
    assert end == f.total_bits
    st = starts.tolist()
    chunk_bits = 8 * C
    for c in range(f.num_blocks * T):
        begin = c * chunk_bits
        if begin >= f.total_bits:
            want = 0
        else:
            later = [s for s in st if s >= begin]
            want = (later[0] if later else f.total_bits) - begin
        assert f.gaps[c] == want
        assert 0 <= want <= 31
    for b in range(f.num_blocks + 1):
        want = sum(1 for s in st if s < b * chunk_bits * T) if b < f.num_blocks else f.n
        assert f.block_out_pos[b] == want
    per_chunk = [0] * (f.num_blocks * T)
    for s in st:
        per_chunk[s // chunk_bits] += 1
    assert f.max_chunk_elems == max(per_chunk)
    assert f.max_warp_elems == max(sum(per_chunk[g:g + 32]) for g in range(0, len(per_chunk), 32))
    assert f.chunk_counts[: len(per_chunk)].tolist() == per_chunk
    assert not f.chunk_counts[len(per_chunk):].any()
    # packed gaps: 5-bit fields, MSB first
    bits = np.unpackbits(f.gaps_packed)
    for c in range(f.num_blocks * T):
        v = int("".join(str(int(x)) for x in bits[5 * c:5 * c + 5]), 2)
        assert v == f.gaps[c]
    # decode from a sample of chunk starts
    idx = 0
    for c in range(0, f.num_blocks * T, 37):
        begin = c * chunk_bits + int(f.gaps[c])
        if begin >= f.total_bits:
            continue
        idx = st.index(begin)
        out, _, _ = oracle.decode(f.bitstream, f.code_lengths,
                                  f.sign_mantissa[idx:], 5, start_bit=begin)
        assert np.array_equal(out, w[idx:idx + 5])


# -------------------------------------------------------------------------
# Round trips and the size claim

@pytest.mark.parametrize("n", [0, 1, 2, 31, 32, 33, 127, 4095, 6399, 6400, 6401])
def test_small_and_ragged_sizes_round_trip(n):
    w = workloads.as_numpy_u16(workloads.gaussian_bf16(n, 0.02, 11 + n))
    f, out = oracle.roundtrip(w, 8, 256)
    assert np.array_equal(out, w)
    assert f.block_out_pos[-1] == n
    if n == 0:
        assert f.num_blocks == 0 and f.total_bits == 0


def test_all_zero_tensor_single_symbol():
    w = np.zeros(100000, np.uint16)
    f, out = oracle.roundtrip(w, 8, 256)
    assert np.array_equal(out, w)
    assert f.total_bits == 100000 and f.max_len == 1
    assert f.max_block_elems == 8 * 8 * 256  # one bit per element


@pytest.mark.parametrize("name", ["single_matrix", "block_scaled", "adversarial",
                                  "fibonacci"])
def test_workloads_round_trip(name):
    if name == "single_matrix":
        ws = [workloads.single_matrix(0)]
    elif name == "block_scaled":
        ws = [t.bits for t in workloads.block_tensors(1, scale=32)]
    elif name == "adversarial":
        ws = [workloads.adversarial_mix(1 << 21, 3)]
    else:
        ws = [workloads.fibonacci_exponents(0)]
    for t in ws:
        w = workloads.as_numpy_u16(t)
        f, out = oracle.roundtrip(w, 8, 256)
        assert np.array_equal(out, w)
        if name == "fibonacci":
            assert f.max_len == 32 and f.num_luts >= 4


def test_size_claim_about_eleven_bits_per_weight():
    """~11 bits/weight, ~30% smaller ("DFloat11无损压缩技术" §2.2 item 2);
    Gaussian weights land at ~10.6 + metadata."""
    cases = [workloads.single_matrix(0)] + \
            [t.bits for t in workloads.block_tensors(2, scale=16)]
    for t in cases:
        w = workloads.as_numpy_u16(t)
        f = oracle.encode(w, 8, 256)
        total = (f.total_bits + 8 * f.n + 5 * f.num_blocks * 256 +
                 32 * (f.num_blocks + 1) + 32 * 256 * f.num_luts + 8 * 256)
        bpw = total / f.n
        assert 10.5 <= bpw <= 11.2, bpw


# --- the matrix-vector product (oracle.gemv) --------------------------------

def test_bf16_widening_hand_checked_values():
    words = np.array([0x3F80, 0xC000, 0x0001, 0x7F80, 0x8000, 0x3E80], np.uint16)
    got = oracle.bf16_to_f64(words)
    assert got[0] == 1.0 and got[1] == -2.0
    assert got[2] == 2.0 ** -133  # smallest positive subnormal: 2^-126 * 2^-7
    assert math.isinf(got[3]) and got[3] > 0
    assert got[4] == 0.0 and math.copysign(1.0, got[4]) == -1.0
    assert got[5] == 0.25


def test_bf16_widening_is_exact_on_every_finite_pattern():
    w = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = oracle.bf16_to_f64(w)
    fin = np.isfinite(f)
    back = (f[fin].astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(back, w[fin])
    assert np.all((f[fin].astype(np.float32).view(np.uint32) & 0xFFFF) == 0)


def _exact_value(word: int):
    """A finite BF16 word as an exact rational, from its fields."""
    from fractions import Fraction
    s, e, m = word >> 15, (word >> 7) & 0xFF, word & 0x7F
    v = Fraction(m, 128) * Fraction(2) ** -126 if e == 0 else \
        (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)
    return -v if s else v


@pytest.mark.parametrize("rows,cols,batch,seed", [(3, 16, 1, 0), (5, 32, 2, 1), (2, 48, 3, 2)])
def test_gemv_matches_exact_rational_sums(rows, cols, batch, seed):
    rng = np.random.default_rng(seed)
    w = (np.float32(rng.normal(0, 0.05, rows * cols)).view(np.uint32) >> 16).astype(np.uint16)
    x = (np.float32(rng.normal(0, 1.0, batch * cols)).view(np.uint32) >> 16).astype(np.uint16)
    f = oracle.encode(w, 8, 128)
    y = oracle.gemv(f.bitstream, f.code_lengths, f.sign_mantissa, f.n, cols, x)
    assert y.shape == (batch, rows)
    for b in range(batch):
        for r in range(rows):
            terms = [_exact_value(int(w[r * cols + c])) * _exact_value(int(x[b * cols + c]))
                     for c in range(cols)]
            exact = sum(terms)
            bound = cols * 2.0 ** -53 * float(sum(abs(t) for t in terms))
            assert abs(y[b, r] - float(exact)) <= bound + 1e-300


def test_gemv_one_hot_activations_return_weight_columns():
    rng = np.random.default_rng(7)
    rows, cols = 6, 32
    w = (np.float32(rng.normal(0, 0.02, rows * cols)).view(np.uint32) >> 16).astype(np.uint16)
    f = oracle.encode(w, 8, 128)
    W = oracle.bf16_to_f64(w).reshape(rows, cols)
    for j in (0, 5, 31):
        x = np.zeros(cols, np.uint16)
        x[j] = 0x3F80  # 1.0
        y = oracle.gemv(f.bitstream, f.code_lengths, f.sign_mantissa, f.n, cols, x)
        assert np.array_equal(y[0], W[:, j])  # column j, row by row: no transpose slip


def test_gemv_interleaved_stream_equals_row_major():
    """The same matrix encoded in the interleaved order (built here by
    explicit index loops) gives the row-major result exactly."""
    rng = np.random.default_rng(9)
    rows, cols, R = 16, 48, 8
    w = (np.float32(rng.normal(0, 0.05, rows * cols)).view(np.uint32) >> 16).astype(np.uint16)
    W = w.reshape(rows, cols)
    inter = np.zeros_like(w)
    j = 0
    for rb in range(rows // R):
        for cg in range(cols // 16):
            for r in range(R):
                for k in range(16):
                    inter[j] = W[rb * R + r, cg * 16 + k]
                    j += 1
    x = (np.float32(rng.normal(0, 1, 2 * cols)).view(np.uint32) >> 16).astype(np.uint16)
    fa, fb = oracle.encode(w, 8, 128), oracle.encode(inter, 8, 128)
    ya = oracle.gemv(fa.bitstream, fa.code_lengths, fa.sign_mantissa, fa.n, cols, x)
    yb = oracle.gemv(fb.bitstream, fb.code_lengths, fb.sign_mantissa, fb.n, cols, x, interleave=R)
    assert np.array_equal(ya, yb)
