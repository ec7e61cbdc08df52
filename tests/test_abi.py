"""The C ABI: libdf11.so loads, exports every function include/df11.h
declares, and rejects bad arguments on the host before touching the GPU.
No call here launches a kernel."""
import ctypes
import os
import re
import subprocess

import pytest

import huffman_decode_df11_b200 as df11

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(df11_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_function():
    lib = df11.lib()
    declared = _declared_functions()
    assert {"df11_decode", "df11_decode_batched", "df11_build"} <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = declared - exported
    assert not missing, missing
    for name in declared:
        getattr(lib, name)  # resolvable through ctypes


def test_struct_layouts_match_header():
    assert ctypes.sizeof(df11.Params) == 48
    assert ctypes.sizeof(df11.TensorDesc) == 9 * 8 + 48


def _params(**kw):
    p = df11.Params(n=1000, total_bits=2600, chunk_bytes=8, threads_per_block=256,
                    num_blocks=1, num_luts=1, max_block_elems=1000, max_len=10,
                    max_chunk_elems=40, max_warp_elems=1000)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


FAKE = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced


def _call(p, n=None, ptrs=None, err=None):
    ptrs = ptrs or [FAKE] * 7
    return df11.lib().df11_decode(*ptrs, p.n if n is None else n, ctypes.byref(p), err, None)


def test_host_validation_errors():
    L = df11.lib()
    assert L.df11_decode(*[FAKE] * 7, 10, None, None, None) == 1           # NULL params
    assert _call(_params(), n=999) == 7                                      # n mismatch
    assert _call(_params(n=0, total_bits=0, num_blocks=0)) == 0             # empty: no-op
    assert _call(_params(), ptrs=[FAKE] * 6 + [0]) == 1                      # NULL out
    assert _call(_params(), ptrs=[FAKE + 8] + [FAKE] * 6) == 2               # misaligned
    assert _call(_params(), err=FAKE + 2) == 2                               # misaligned err
    assert _call(_params(chunk_bytes=12)) == 4                               # unsupported C
    assert _call(_params(threads_per_block=384)) == 4                        # unsupported T
    assert _call(_params(num_blocks=2)) == 3                                 # wrong block count
    assert _call(_params(total_bits=999)) == 3                               # < 1 bit/element
    assert _call(_params(total_bits=40000)) == 3                             # > 32 bits/element
    assert _call(_params(num_luts=0)) == 3
    assert _call(_params(max_block_elems=20000)) == 3
    assert _call(_params(max_chunk_elems=65)) == 3                           # > 8*C
    assert _call(_params(max_warp_elems=0)) == 3
    assert _call(_params(max_warp_elems=32 * 40 + 1)) == 3                   # > 32*max_chunk
    assert _call(_params(max_len=33)) == 3
    assert _call(_params(n=1 << 32, total_bits=1 << 34, num_blocks=1 << 20)) == 6


def test_batched_host_validation():
    L = df11.lib()
    assert L.df11_decode_batched(None, 0, None, None) == 0
    assert L.df11_decode_batched(None, -1, None, None) == 7
    assert L.df11_decode_batched(None, 1, None, None) == 1
    a = df11.TensorDesc(*[FAKE] * 8, None, _params())
    b = df11.TensorDesc(*[FAKE] * 8, None, _params(chunk_bytes=4, total_bits=2600,
                                                      num_blocks=1, max_chunk_elems=30,
                                                      max_warp_elems=900))
    arr = (df11.TensorDesc * 2)(a, b)
    assert L.df11_decode_batched(arr, 2, None, None) == 7  # mixed (C, T)
    c = df11.TensorDesc(*[FAKE] * 8, FAKE + 8, _params())  # misaligned decode table
    assert L.df11_decode_batched(ctypes.byref(c), 1, None, None) == 2


def test_decode_table_host_validation():
    L = df11.lib()
    assert L.df11_build_decode_table(None, FAKE, 1, FAKE, None) == 1
    assert L.df11_build_decode_table(FAKE, FAKE, 1, None, None) == 1
    assert L.df11_build_decode_table(FAKE + 4, FAKE, 1, FAKE, None) == 2
    assert L.df11_build_decode_table(FAKE, FAKE, 1, FAKE + 8, None) == 2
    assert L.df11_build_decode_table(FAKE, FAKE, 0, FAKE, None) == 3
    assert L.df11_build_decode_table(FAKE, FAKE, 1 << 24, FAKE, None) == 3


def test_device_builder_host_validation():
    """Phase 1 rejects bad arguments before any CUDA call; phase 2 rejects a
    NULL handle; freeing NULL is a no-op."""
    L = df11.lib()
    p = df11.Params()
    lens = (ctypes.c_uint8 * 256)()
    lp = ctypes.cast(lens, ctypes.c_void_p)
    h = ctypes.c_void_p(123)
    assert L.df11_gpu_build_begin(None, 10, 24, 256, None, ctypes.byref(p), lp,
                                  ctypes.byref(h)) == 1
    assert h.value is None  # cleared even on error
    assert L.df11_gpu_build_begin(FAKE, 10, 24, 256, None, None, lp, ctypes.byref(h)) == 1
    assert L.df11_gpu_build_begin(FAKE, 10, 6, 256, None, ctypes.byref(p), lp,
                                  ctypes.byref(h)) == 7   # C not a multiple of 4
    assert L.df11_gpu_build_begin(FAKE, 10, 32, 256, None, ctypes.byref(p), lp,
                                  ctypes.byref(h)) == 7   # counts would not fit a byte
    assert L.df11_gpu_build_begin(FAKE, 10, 24, 200, None, ctypes.byref(p), lp,
                                  ctypes.byref(h)) == 7
    assert L.df11_gpu_build_begin(FAKE, 1 << 32, 24, 256, None, ctypes.byref(p), lp,
                                  ctypes.byref(h)) == 6
    assert L.df11_gpu_build_begin(FAKE + 1, 10, 24, 256, None, ctypes.byref(p), lp,
                                  ctypes.byref(h)) == 2
    assert L.df11_gpu_build_finish(None, *[FAKE] * 8, ctypes.byref(p), None) == 1
    L.df11_gpu_build_free(None)
    with pytest.raises(ValueError):
        df11.compress_on_device(df11.torch.zeros(4, dtype=df11.torch.int16))


def test_build_layout_places_every_buffer():
    """df11_gpu_build_layout (host only): the seven buffers of each tensor
    with the sizes the header lists, at 256-byte offsets in order, none
    overlapping, none below 16 bytes, and the total covering the last."""
    L = df11.lib()
    ps = [_params(n=1000, num_blocks=1, num_luts=1),
          _params(n=0, num_blocks=0, num_luts=1, chunk_bytes=24, threads_per_block=512),
          _params(n=123_457, num_blocks=37, num_luts=4, chunk_bytes=12, threads_per_block=128)]
    arr = (df11.Params * len(ps))(*ps)
    offs = (ctypes.c_uint64 * (7 * len(ps)))()
    sizes = (ctypes.c_uint64 * (7 * len(ps)))()
    total = L.df11_gpu_build_layout(arr, len(ps), offs, sizes)
    end = 0
    for i, p in enumerate(ps):
        chunks = p.num_blocks * p.threads_per_block
        want = [chunks * p.chunk_bytes + 16, chunks * 5 // 8 + 16, chunks + 16,
                4 * (p.num_blocks + 1), 4 * 256 * p.num_luts, 256, -(-p.n // 16) * 16]
        for j, w in enumerate(want):
            o, sz = offs[7 * i + j], sizes[7 * i + j]
            assert sz == w
            assert o % 256 == 0 and o >= end
            end = o + max(sz, 16)
    assert end <= total < end + 256
    assert L.df11_gpu_build_layout(arr, len(ps), None, None) == total
    assert L.df11_gpu_build_layout(arr, 0, None, None) == 0
    assert L.df11_gpu_build_layout(None, 3, None, None) == 0
    assert L.df11_gpu_build_layout(arr, -1, None, None) == 0


def test_batched_builder_host_validation():
    """The batched builder phases reject bad arguments before any CUDA
    call, and clear the handles they would return."""
    L = df11.lib()
    vp = ctypes.c_void_p
    ptrs = (vp * 2)(FAKE, FAKE)
    ns = (ctypes.c_uint64 * 2)(100, 200)
    params = (df11.Params * 2)()
    lens = (ctypes.c_uint8 * 512)()
    handles = (vp * 2)(123, 456)
    lp = ctypes.cast(lens, vp)
    assert L.df11_gpu_build_begin_batched(ptrs, ns, 0, 24, 256, None, params, lp, handles) == 0
    assert L.df11_gpu_build_begin_batched(ptrs, ns, -1, 24, 256, None, params, lp, handles) == 7
    assert L.df11_gpu_build_begin_batched(None, ns, 2, 24, 256, None, params, lp, handles) == 1
    assert handles[0] is None and handles[1] is None  # cleared on error
    assert L.df11_gpu_build_begin_batched(ptrs, ns, 2, 6, 256, None, params, lp, handles) == 7
    bad = (vp * 2)(FAKE, FAKE + 1)
    assert L.df11_gpu_build_begin_batched(bad, ns, 2, 24, 256, None, params, lp, handles) == 2
    big = (ctypes.c_uint64 * 2)(100, 1 << 32)
    assert L.df11_gpu_build_begin_batched(ptrs, big, 2, 24, 256, None, params, lp, handles) == 6
    assert L.df11_gpu_build_finish_batched(None, 2, ptrs, None, params, None) == 1
    assert L.df11_gpu_build_finish_batched(handles, 0, ptrs, None, params, None) == 0
    assert L.df11_gpu_build_finish_batched(handles, -1, ptrs, None, params, None) == 7


def test_gemv_host_validation():
    """df11_decode_gemv rejects bad arguments before any CUDA call."""
    L = df11.lib()
    t = (df11.TensorDesc * 1)(df11.TensorDesc(*[FAKE] * 7, None, None,
                                              _params(n=4096 * 64, chunk_bytes=24)))
    def op(**kw):
        f = dict(x=FAKE, y=FAKE, cols=4096, batch=1, x_stride=4096, y_stride=64, accumulate=0,
                 pad=0)
        f.update(kw)
        return (df11.GemvOp * 1)(df11.GemvOp(**f))
    assert L.df11_decode_gemv(t, op(), 0, None, None) == 0
    assert L.df11_decode_gemv(None, op(), 1, None, None) == 1
    assert L.df11_decode_gemv(t, None, 1, None, None) == 1
    assert L.df11_decode_gemv(t, op(), -1, None, None) == 7
    assert L.df11_decode_gemv(t, op(cols=4095), 1, None, None) == 7
    assert L.df11_decode_gemv(t, op(batch=9), 1, None, None) == 7
    assert L.df11_decode_gemv(t, op(y_stride=63), 1, None, None) == 7
    assert L.df11_decode_gemv(t, op(x=FAKE + 2), 1, None, None) == 2
    assert L.df11_decode_gemv(t, op(x=None), 1, None, None) == 1


def test_supported_shapes_and_shared_bytes():
    assert df11.supported(8, 256) and df11.supported(4, 256) and df11.supported(16, 256)
    assert df11.supported(24, 256) and not df11.supported(20, 256)
    assert df11.supported(8, 128) and df11.supported(8, 512)
    assert not df11.supported(12, 256)
    p = _params(max_block_elems=6400, num_luts=4)
    sb = df11.lib().df11_shared_bytes(ctypes.byref(p))
    # tables (16 KB derived table) + two stage slots + exponents + slots
    assert 30_000 < sb < 60_000
    bigger = _params(max_block_elems=12800, num_luts=4)
    assert df11.lib().df11_shared_bytes(ctypes.byref(bigger)) > sb
    assert df11.lib().df11_shared_bytes(ctypes.byref(_params(chunk_bytes=12))) == 0


def test_status_strings():
    L = df11.lib()
    for code in range(9):
        assert L.df11_status_string(code)
    for code in range(6):
        assert L.df11_device_error_string(code)
