"""df11_exponent_histogram: the exponent histogram into the library's static
device counters, with no allocation.

The counts must equal numpy's bincount of the exponent field (bits 7-14) on
every input; repeated calls must leave the device's free memory unchanged
(no allocation, not even from a pool); concurrent calls from several host
threads must each get their own tensor's counts (the library serialises
them on its one buffer).  The host-side argument checks run without a GPU.
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


@gpu
@pytest.mark.parametrize("n", [0, 1, 7, 8, 2047, 2049, 1_000_003, 40_000_000])
def test_counts_match_bincount(cuda, n):
    w = workloads.gaussian_bf16(n, 0.02, 900 + n, device="cuda")
    got = df11.exponent_histogram(w)
    assert np.array_equal(got, _want(workloads.as_numpy_u16(w)))


@gpu
def test_every_pattern_adversarial_and_unaligned(cuda):
    for w in (workloads.all_bf16_patterns("cuda"), workloads.adversarial_mix(1 << 22, 8, "cuda"),
              workloads.fibonacci_exponents(2, "cuda")):
        assert np.array_equal(df11.exponent_histogram(w), _want(workloads.as_numpy_u16(w)))
    base = workloads.gaussian_bf16(300_001, 0.02, 9, device="cuda")
    view = base[5:]  # not 16-byte aligned: the scalar loads
    assert view.data_ptr() % 16
    assert np.array_equal(df11.exponent_histogram(view), _want(workloads.as_numpy_u16(view)))


@gpu
def test_allocates_nothing(cuda):
    w = workloads.gaussian_bf16(10_000_000, 0.02, 4, device="cuda")
    df11.exponent_histogram(w)  # the library and its module are loaded now
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    reserved_before = torch.cuda.memory_reserved()
    for _ in range(20):
        df11.exponent_histogram(w)
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
