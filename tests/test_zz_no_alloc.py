"""df11_exponent_histogram: the exponent histogram with no device
allocation, for callers that cannot allocate device memory (code that runs
where the CUDA allocator must not be entered, or a program whose device
memory is all handed to its own allocator).  Its counters are a fixed
2 KB array in the library's device memory, shared by every call on a device.

This file is collected last on purpose: if the entry point misbehaves, a run
that stops at the first failure has already run every other test.  Its tests
pass alone in a fresh process and after the others.

The bar: on two calls in a row through the C ABI, the counts equal what the
library's allocating entry point computes from the same words
(df11_gpu_build_begin, whose histogram kernel takes its scratch from a memory
pool): its code lengths are non-zero exactly for the counted exponents, and
its stream length is the sum of count x code length, exactly (integers).
They also equal numpy's bincount of the exponent field.  Repeated calls leave
the device's free memory unchanged; concurrent calls from several host
threads each get their own tensor's counts.
"""
import ctypes
import threading

import numpy as np
import pytest
import torch

import workloads

df11 = pytest.importorskip("huffman_decode_df11_b200")


def _want(w_np):
    return np.bincount((w_np.astype(np.int64) >> 7) & 0xFF, minlength=256).astype(np.uint64)


def test_host_argument_errors():
    L = df11.lib()
    hist = np.zeros(256, np.uint64)
    fake = 1 << 20  # never dereferenced
    assert L.df11_exponent_histogram(None, 10, hist.ctypes.data, None) == 1
    assert L.df11_exponent_histogram(fake, 10, None, None) == 1
    assert L.df11_exponent_histogram(fake, 1 << 32, hist.ctypes.data, None) == 6
    assert L.df11_exponent_histogram(fake + 1, 10, hist.ctypes.data, None) == 2
    with pytest.raises(ValueError):
        df11.exponent_histogram(torch.zeros(4, dtype=torch.int16))


gpu = pytest.mark.gpu


@pytest.fixture
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _c_abi_histogram(w: torch.Tensor) -> np.ndarray:
    """One call of the entry point through the C ABI, on the current stream."""
    hist = np.full(256, 0xDEAD, np.uint64)  # every counter must be written
    st = df11.lib().df11_exponent_histogram(
        ctypes.c_void_p(w.data_ptr() if w.numel() else None), w.numel(), hist.ctypes.data,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, df11.lib().df11_status_string(st)
    return hist


def _allocating_entry_point(w: torch.Tensor):
    """df11_gpu_build_begin on the same words: (code lengths, total bits)."""
    L = df11.lib()
    params = df11.Params()
    lens = (ctypes.c_uint8 * 256)()
    handle = ctypes.c_void_p()
    st = L.df11_gpu_build_begin(ctypes.c_void_p(w.data_ptr() if w.numel() else None),
                                w.numel(), 24, 256,
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                ctypes.byref(params), ctypes.cast(lens, ctypes.c_void_p),
                                ctypes.byref(handle))
    assert st == 0, df11.lib().df11_status_string(st)
    L.df11_gpu_build_free(handle)
    torch.cuda.synchronize()
    return np.frombuffer(bytes(lens), np.uint8).astype(np.uint64), int(params.total_bits)


@gpu
@pytest.mark.parametrize("case", ["gaussian", "adversarial", "fibonacci", "patterns", "ragged"])
def test_two_calls_in_a_row_match_the_allocating_entry_point(cuda, case):
    w = {"gaussian": lambda: workloads.gaussian_bf16(4_000_037, 0.02, 3, device="cuda"),
         "adversarial": lambda: workloads.adversarial_mix(1 << 22, 8, "cuda"),
         "fibonacci": lambda: workloads.fibonacci_exponents(2, "cuda"),
         "patterns": lambda: workloads.all_bf16_patterns("cuda"),
         "ragged": lambda: workloads.gaussian_bf16(77, 0.5, 4, device="cuda")}[case]()
    first = _c_abi_histogram(w)
    second = _c_abi_histogram(w)  # the array keeps the last counts: cleared first
    assert np.array_equal(first, second)
    lens, total_bits = _allocating_entry_point(w)
    assert np.array_equal(first > 0, lens > 0)           # the same exponents occur
    assert int((first * lens).sum()) == total_bits       # exact: sum of count x length
    assert int(first.sum()) == w.numel()
    assert np.array_equal(first, _want(workloads.as_numpy_u16(w)))


@gpu
def test_a_different_tensor_after_a_larger_one(cuda):
    big = workloads.gaussian_bf16(3_000_000, 0.02, 11, device="cuda")
    small = workloads.gaussian_bf16(1000, 3.0, 12, device="cuda")
    _c_abi_histogram(big)
    got = _c_abi_histogram(small)  # nothing of the first call's counts remains
    assert np.array_equal(got, _want(workloads.as_numpy_u16(small)))
    assert np.array_equal(_c_abi_histogram(torch.empty(0, dtype=torch.int16, device="cuda")),
                          np.zeros(256, np.uint64))


@gpu
@pytest.mark.parametrize("n", [1, 7, 8, 2047, 2049, 1_000_003, 40_000_000])
def test_counts_match_bincount(cuda, n):
    w = workloads.gaussian_bf16(n, 0.02, 900 + n, device="cuda")
    got = df11.exponent_histogram(w)
    assert np.array_equal(got, _want(workloads.as_numpy_u16(w)))


@gpu
def test_unaligned_view_and_host_memory(cuda):
    base = workloads.gaussian_bf16(300_001, 0.02, 9, device="cuda")
    view = base[5:]  # not 16-byte aligned: the scalar loads
    assert view.data_ptr() % 16
    assert np.array_equal(df11.exponent_histogram(view), _want(workloads.as_numpy_u16(view)))
    host = np.zeros(1024, np.uint16)  # not device memory: refused before any work
    hist = np.zeros(256, np.uint64)
    assert df11.lib().df11_exponent_histogram(host.ctypes.data, 1024, hist.ctypes.data,
                                              None) == 9
    with pytest.raises(ValueError):
        df11.exponent_histogram(base[:300_000].view(100, 3000)[:, ::2])  # needs a copy


@gpu
def test_allocates_nothing(cuda):
    w = workloads.gaussian_bf16(10_000_000, 0.02, 4, device="cuda")
    df11.exponent_histogram(w)  # the library and its module are loaded now
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    reserved_before = torch.cuda.memory_reserved()
    for _ in range(20):
        _c_abi_histogram(w)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before
    assert torch.cuda.memory_reserved() == reserved_before


@gpu
def test_concurrent_calls_get_their_own_counts(cuda):
    ws = [workloads.gaussian_bf16(3_000_000 + 17 * i, 0.01 * (i + 1), 60 + i, device="cuda")
          for i in range(4)]
    wants = [_want(workloads.as_numpy_u16(w)) for w in ws]
    results = [[] for _ in ws]

    def run(i):
        s = torch.cuda.Stream()
        for _ in range(5):
            results[i].append(df11.exponent_histogram(ws[i], stream=s))

    threads = [threading.Thread(target=run, args=(i,)) for i in range(len(ws))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    for want, got in zip(wants, results):
        assert len(got) == 5
        for g in got:
            assert np.array_equal(g, want)
