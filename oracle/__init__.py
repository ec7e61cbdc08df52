"""CPU oracle for DFloat11 (DF11) Huffman-coded BF16 weights.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  The
product package never does, and this module never imports the product package:
the two share no code.  The arithmetic lives in ``oracle.c`` (plain C,
single-threaded, bit-at-a-time); this file only compiles it and marshals numpy
arrays through ctypes.

Functions and what pins them (tests/test_oracle_pins.py, tests/golden/):

==========================  ==================================================
split / histogram           exact BF16 round trip over all 65,536 bit patterns
huffman_lengths             brute-force optimum on small alphabets; Kraft
                            equality; entropy bound H <= avg < H + 1; the
                            tie order on hand-worked tied histograms
package_merge_lengths       brute-force optimum of the length-limited problem;
                            equal total cost to Huffman when the limit is
                            slack; leaf-first ties on hand-worked cases
code_lengths                32-bit cap reached exactly on Fibonacci weights
canonical_codes             RFC 1951 section 3.2.2 worked example; prefix-free
build_luts                  every entry re-derived by brute-force parsing
encode / decode             round trip on every synthetic workload; decoded
                            hand-written bit strings in tests/golden/
metadata_from_starts        brute-force gap / block position definitions
bf16_to_f64                 hand-checked values (1, -2, the smallest subnormal,
                            infinity); every finite pattern widens and narrows
                            back exactly
gemv                        exact rational sums (fractions.Fraction) of tiny
                            products; one-hot activations return the decoded
                            weight columns exactly; an interleaved stream of
                            a matrix gives the row-major stream's result
==========================  ==================================================

No function is left "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

MAX_LEN = 32


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, no GPU needed)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-Wall", "-Wextra", "-shared", "-fPIC",
             _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class _Format(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_uint64),
        ("total_bits", ctypes.c_uint64),
        ("chunk_bytes", ctypes.c_uint32),
        ("threads_per_block", ctypes.c_uint32),
        ("num_blocks", ctypes.c_uint32),
        ("num_luts", ctypes.c_uint32),
        ("max_block_elems", ctypes.c_uint32),
        ("max_len", ctypes.c_uint32),
        ("max_chunk_elems", ctypes.c_uint32),
        ("max_warp_elems", ctypes.c_uint32),
        ("code_lengths", ctypes.c_uint8 * 256),
        ("codes", ctypes.c_uint32 * 256),
        ("bitstream", ctypes.POINTER(ctypes.c_uint8)),
        ("bitstream_bytes", ctypes.c_uint64),
        ("gaps", ctypes.POINTER(ctypes.c_uint8)),
        ("gaps_packed", ctypes.POINTER(ctypes.c_uint8)),
        ("gaps_bytes", ctypes.c_uint64),
        ("block_out_pos", ctypes.POINTER(ctypes.c_uint32)),
        ("luts", ctypes.POINTER(ctypes.c_uint32)),
        ("sign_mantissa", ctypes.POINTER(ctypes.c_uint8)),
        ("sm_bytes", ctypes.c_uint64),
        ("chunk_counts", ctypes.POINTER(ctypes.c_uint8)),
        ("chunk_counts_bytes", ctypes.c_uint64),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        lib.oracle_split.argtypes = [u16p, ctypes.c_uint64, u8p, u8p]
        lib.oracle_histogram.argtypes = [u8p, ctypes.c_uint64, u64p]
        lib.oracle_huffman_lengths.argtypes = [u64p, u8p]
        lib.oracle_huffman_lengths.restype = ctypes.c_int
        lib.oracle_package_merge_lengths.argtypes = [u64p, ctypes.c_int, u8p]
        lib.oracle_package_merge_lengths.restype = ctypes.c_int
        lib.oracle_code_lengths.argtypes = [u64p, u8p]
        lib.oracle_code_lengths.restype = ctypes.c_int
        lib.oracle_canonical_codes.argtypes = [u8p, u32p]
        lib.oracle_build_luts.argtypes = [u8p, u32p, u32p, ctypes.c_int]
        lib.oracle_build_luts.restype = ctypes.c_int
        lib.oracle_encode.argtypes = [u16p, ctypes.c_uint64, ctypes.c_uint32,
                                      ctypes.c_uint32, ctypes.POINTER(_Format)]
        lib.oracle_encode.restype = ctypes.c_int
        lib.oracle_format_free.argtypes = [ctypes.POINTER(_Format)]
        lib.oracle_decode.argtypes = [u8p, ctypes.c_uint64, ctypes.c_uint64,
                                      u8p, u8p, ctypes.c_uint64, u16p, u64p]
        lib.oracle_decode.restype = ctypes.c_uint64
        lib.oracle_metadata_from_starts.argtypes = [
            u64p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
            ctypes.c_uint32, ctypes.c_uint32, u8p, u32p]
        lib.oracle_pack_gaps.argtypes = [u8p, ctypes.c_uint64, u8p]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _u16(w) -> np.ndarray:
    a = np.ascontiguousarray(w)
    if a.dtype != np.uint16:
        a = a.view(np.uint16) if a.dtype.itemsize == 2 else a.astype(np.uint16)
    return a


@dataclass
class OracleFormat:
    """Everything the oracle encoder emits, as numpy arrays."""
    n: int
    total_bits: int
    chunk_bytes: int
    threads_per_block: int
    num_blocks: int
    num_luts: int
    max_block_elems: int
    max_len: int
    max_chunk_elems: int
    max_warp_elems: int
    code_lengths: np.ndarray   # uint8[256]
    codes: np.ndarray          # uint32[256]
    bitstream: np.ndarray      # uint8[num_blocks*T*C + 16]
    gaps: np.ndarray           # uint8[num_blocks*T], unpacked
    gaps_packed: np.ndarray    # uint8[num_blocks*T*5/8 + 16]
    block_out_pos: np.ndarray  # uint32[num_blocks + 1]
    luts: np.ndarray           # uint32[num_luts*256]
    sign_mantissa: np.ndarray  # uint8[roundup(n, 16)]
    chunk_counts: np.ndarray   # uint8[num_blocks*T + 16]


def split(w):
    w = _u16(w)
    n = w.size
    e = np.empty(n, np.uint8)
    s = np.empty(n, np.uint8)
    _load().oracle_split(_ptr(w, ctypes.c_uint16), n, _ptr(e, ctypes.c_uint8),
                         _ptr(s, ctypes.c_uint8))
    return e, s


def histogram(exps) -> np.ndarray:
    e = np.ascontiguousarray(exps, dtype=np.uint8)
    h = np.zeros(256, np.uint64)
    _load().oracle_histogram(_ptr(e, ctypes.c_uint8), e.size,
                             _ptr(h, ctypes.c_uint64))
    return h


def _hist_arr(hist) -> np.ndarray:
    h = np.zeros(256, np.uint64)
    hist = np.asarray(hist, dtype=np.uint64)
    h[: hist.size] = hist
    return h


def huffman_lengths(hist):
    h = _hist_arr(hist)
    out = np.zeros(256, np.uint8)
    longest = _load().oracle_huffman_lengths(_ptr(h, ctypes.c_uint64),
                                             _ptr(out, ctypes.c_uint8))
    return out, longest


def package_merge_lengths(hist, max_len: int):
    h = _hist_arr(hist)
    out = np.zeros(256, np.uint8)
    longest = _load().oracle_package_merge_lengths(
        _ptr(h, ctypes.c_uint64), max_len, _ptr(out, ctypes.c_uint8))
    return out, longest


def code_lengths(hist):
    h = _hist_arr(hist)
    out = np.zeros(256, np.uint8)
    longest = _load().oracle_code_lengths(_ptr(h, ctypes.c_uint64),
                                          _ptr(out, ctypes.c_uint8))
    return out, longest


def canonical_codes(lengths) -> np.ndarray:
    ln = np.zeros(256, np.uint8)
    lengths = np.asarray(lengths, dtype=np.uint8)
    ln[: lengths.size] = lengths
    codes = np.zeros(256, np.uint32)
    _load().oracle_canonical_codes(_ptr(ln, ctypes.c_uint8),
                                   _ptr(codes, ctypes.c_uint32))
    return codes


def build_luts(lengths, codes=None) -> np.ndarray:
    ln = np.zeros(256, np.uint8)
    lengths = np.asarray(lengths, dtype=np.uint8)
    ln[: lengths.size] = lengths
    if codes is None:
        codes = canonical_codes(ln)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    lib = _load()
    count = lib.oracle_build_luts(_ptr(ln, ctypes.c_uint8),
                                  _ptr(codes, ctypes.c_uint32), None, 0)
    luts = np.zeros(count * 256, np.uint32)
    lib.oracle_build_luts(_ptr(ln, ctypes.c_uint8), _ptr(codes, ctypes.c_uint32),
                          _ptr(luts, ctypes.c_uint32), count)
    return luts


def _copy(ptr, count, dtype):
    if count == 0:
        return np.zeros(0, dtype)
    ctype = np.ctypeslib.as_ctypes_type(dtype)
    buf = ctypes.cast(ptr, ctypes.POINTER(ctype * count)).contents
    return np.frombuffer(buf, dtype=dtype, count=count).copy()


def encode(w, chunk_bytes: int = 8, threads_per_block: int = 256) -> OracleFormat:
    """Encode BF16 words (any 2-byte array) into the DF11 chunked format."""
    w = _u16(w).reshape(-1)
    f = _Format()
    lib = _load()
    rc = lib.oracle_encode(_ptr(w, ctypes.c_uint16), w.size, chunk_bytes,
                           threads_per_block, ctypes.byref(f))
    if rc != 0:
        raise ValueError("oracle_encode rejected its arguments")
    try:
        chunks = f.num_blocks * f.threads_per_block
        out = OracleFormat(
            n=f.n, total_bits=f.total_bits, chunk_bytes=f.chunk_bytes,
            threads_per_block=f.threads_per_block, num_blocks=f.num_blocks,
            num_luts=f.num_luts, max_block_elems=f.max_block_elems,
            max_len=f.max_len, max_chunk_elems=f.max_chunk_elems,
            max_warp_elems=f.max_warp_elems,
            code_lengths=np.frombuffer(bytes(f.code_lengths), np.uint8).copy(),
            codes=np.array(list(f.codes), dtype=np.uint32),
            bitstream=_copy(f.bitstream, f.bitstream_bytes, np.uint8),
            gaps=_copy(f.gaps, chunks, np.uint8),
            gaps_packed=_copy(f.gaps_packed, f.gaps_bytes, np.uint8),
            block_out_pos=_copy(f.block_out_pos, f.num_blocks + 1, np.uint32),
            luts=_copy(f.luts, f.num_luts * 256, np.uint32),
            sign_mantissa=_copy(f.sign_mantissa, f.sm_bytes, np.uint8),
            chunk_counts=_copy(f.chunk_counts, f.chunk_counts_bytes, np.uint8),
        )
    finally:
        lib.oracle_format_free(ctypes.byref(f))
    return out


def decode(bitstream, code_lengths, sign_mantissa, count: int,
           start_bit: int = 0, want_starts: bool = False):
    """Bit-serial decode of `count` codewords from `start_bit`.

    Returns (bf16 words as uint16, end bit, starts or None)."""
    bs = np.ascontiguousarray(bitstream, dtype=np.uint8)
    ln = np.ascontiguousarray(code_lengths, dtype=np.uint8)
    sm = np.ascontiguousarray(sign_mantissa, dtype=np.uint8)
    if sm.size < count:
        raise ValueError("sign_mantissa shorter than count")
    out = np.zeros(max(count, 1), np.uint16)
    starts = np.zeros(max(count, 1), np.uint64) if want_starts else None
    end = _load().oracle_decode(
        _ptr(bs, ctypes.c_uint8), bs.size, start_bit, _ptr(ln, ctypes.c_uint8),
        _ptr(sm, ctypes.c_uint8), count, _ptr(out, ctypes.c_uint16),
        _ptr(starts, ctypes.c_uint64) if starts is not None else None)
    if end == 2 ** 64 - 1:
        raise ValueError("invalid bitstream")
    return out[:count], int(end), (starts[:count] if starts is not None else None)


def metadata_from_starts(starts, n, total_bits, chunk_bytes, threads_per_block,
                         num_blocks):
    st = np.ascontiguousarray(starts if n else np.zeros(1), dtype=np.uint64)
    gaps = np.zeros(max(num_blocks * threads_per_block, 1), np.uint8)
    pos = np.zeros(num_blocks + 1, np.uint32)
    _load().oracle_metadata_from_starts(
        _ptr(st, ctypes.c_uint64), n, total_bits, chunk_bytes,
        threads_per_block, num_blocks, _ptr(gaps, ctypes.c_uint8),
        _ptr(pos, ctypes.c_uint32))
    return gaps[: num_blocks * threads_per_block], pos


def pack_gaps(gaps) -> np.ndarray:
    g = np.ascontiguousarray(gaps, dtype=np.uint8)
    out = np.zeros(g.size * 5 // 8 + 16, np.uint8)
    _load().oracle_pack_gaps(_ptr(g, ctypes.c_uint8), g.size,
                             _ptr(out, ctypes.c_uint8))
    return out


def roundtrip(w, chunk_bytes: int = 8, threads_per_block: int = 256):
    """encode then decode; returns (format, decoded uint16)."""
    f = encode(w, chunk_bytes, threads_per_block)
    out, end, _ = decode(f.bitstream, f.code_lengths, f.sign_mantissa, f.n)
    if end != f.total_bits:
        raise ValueError("decode did not end at the last encoded bit")
    return f, out


def bf16_to_f64(words) -> np.ndarray:
    """BF16 bit patterns (any 2-byte array) as float64: a BF16 word is the top
    half of the float32 with the same bits, and float32 widens to float64
    exactly."""
    u = np.ascontiguousarray(words).view(np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):  # NaN patterns stay NaN
        return u.view(np.float32).astype(np.float64)


def gemv(bitstream, code_lengths, sign_mantissa, n: int, cols: int, x,
         interleave: int = 1) -> np.ndarray:
    """y = W x for the tensor W that the stream decodes to, taken as
    (n / cols) x cols (a weight applied right after its decode,
    "DFloat11无损压缩技术" (jsqmd.com) §2.2 item 3), and BF16 activations x
    (batch x cols, or cols).  The stream is row-major, or with `interleave`
    = R > 1 holds, for each block of R rows and each group of 16 columns,
    the R rows' 16 elements one after another (the library's option for its
    fused product); the element of row r, column c is then at
    ((r // R * (cols // 16) + c // 16) * R + r % R) * 16 + c % 16.
    Float64 throughout: the decoded weights and the activations widen
    exactly, and the product is one library matmul.  Returns float64 of
    shape (batch, n / cols)."""
    if cols <= 0 or n % cols:
        raise ValueError("cols must divide n")
    rows = n // cols
    w, end, _ = decode(bitstream, code_lengths, sign_mantissa, n)
    if interleave > 1:
        R = interleave
        if rows % R or cols % 16:
            raise ValueError("interleave needs rows a multiple of R and cols of 16")
        r = np.arange(rows)[:, None]
        c = np.arange(cols)[None, :]
        pos = ((r // R * (cols // 16) + c // 16) * R + r % R) * 16 + c % 16
        w = w[pos]
    W = bf16_to_f64(w).reshape(rows, cols)
    X = bf16_to_f64(np.ascontiguousarray(x)).reshape(-1, cols)
    return X @ W.T
