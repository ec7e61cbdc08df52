"""Failure detection of the decode kernels without a GPU fault.

Every wait in the decode kernels is bounded.  The host withholds the stage
copies of one launch (df11_test_withhold_copies: the producer issues none),
so that the consumers' waits run out: the launch must report
DF11_DEV_ERR_TIMEOUT in the error word, leave no copy in flight, and the
next decode on the same context must be bit-exact.  Nothing here traps,
faults or hangs: the waits end after a few thousand polls.
"""
import numpy as np
import pytest
import torch

import workloads

df11 = pytest.importorskip("huffman_decode_df11_b200")

TIMEOUT = 4  # DF11_DEV_ERR_TIMEOUT


def test_hook_rejects_out_of_range_arguments():
    L = df11.lib()
    assert L.df11_test_withhold_copies(-1, 100) == 7
    assert L.df11_test_withhold_copies(1, 0) == 7
    assert L.df11_test_withhold_copies(1, (1 << 20) + 1) == 7
    assert L.df11_test_withhold_copies(0, 100) == 0  # nothing withheld


@pytest.fixture
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    yield
    df11.lib().df11_test_withhold_copies(0, 1 << 20)


def _tensors(k):
    ws = [workloads.gaussian_bf16(300_000 + 70_001 * i, 0.02, 40 + i) for i in range(k)]
    return ws, [df11.to_device(df11.compress(w)) for w in ws]


@pytest.mark.gpu
@pytest.mark.parametrize("k", [1, 5])
def test_withheld_copies_time_out_and_the_next_decode_is_exact(cuda, k):
    ws, ds = _tensors(k)
    outs = [df11.empty_output(d) for d in ds]
    err = df11.new_error_word()
    L = df11.lib()
    assert L.df11_test_withhold_copies(1, 2000) == 0
    df11.decode_batched(ds, outs, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == TIMEOUT
    with pytest.raises(df11.Df11Error, match="TIMEOUT"):
        df11.check_device_error(err)
    # the hook covered one launch only; the context is usable and exact
    err.zero_()
    df11.decode_batched(ds, outs, err=err)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for o, w in zip(outs, ws):
        assert np.array_equal(o.view(torch.int16).cpu().numpy(), w.numpy())


@pytest.mark.gpu
def test_withheld_copies_in_the_middle_of_a_layer_loop(cuda):
    """A timeout in one launch of a sequence (dependent launches on one
    stream) is reported, and the launches after it decode exactly."""
    ws, ds = _tensors(3)
    outs = [df11.empty_output(d) for d in ds]
    err = df11.new_error_word()
    got = []
    for i, (d, o) in enumerate(zip(ds, outs)):
        if i == 1:
            assert df11.lib().df11_test_withhold_copies(1, 2000) == 0
        df11.decode(d, o, err=err)
        got.append(o.clone())
    torch.cuda.synchronize()
    assert int(err.item()) == TIMEOUT
    for i in (0, 2):
        assert np.array_equal(got[i].view(torch.int16).cpu().numpy(), ws[i].numpy())


@pytest.mark.gpu
def test_buffers_that_are_not_device_memory_are_refused(cuda):
    """A call whose buffers are not memory of the current device returns
    DF11_ERR_DEVICE before anything is queued (a kernel would otherwise read
    host or another GPU's memory)."""
    import ctypes
    ws, ds = _tensors(2)
    outs = [df11.empty_output(d) for d in ds]
    host_out = np.zeros(ds[1].n + 8, np.uint16)
    descs = (df11.TensorDesc * 2)(ds[0].desc(outs[0]), ds[1].desc(outs[1]))
    descs[1].out_bf16 = (host_out.ctypes.data + 15) // 16 * 16
    err = df11.new_error_word()
    outs[0].fill_(0)
    st = df11.lib().df11_decode_batched(descs, 2, err.data_ptr(), None)
    torch.cuda.synchronize()
    assert st == 9  # DF11_ERR_DEVICE
    assert int(err.item()) == 0
    assert not outs[0].view(torch.int16).any()  # nothing was decoded
    assert not host_out.any()
    hist = np.zeros(256, np.uint64)
    bad = torch.zeros(16, dtype=torch.int16).pin_memory()  # host memory
    assert df11.lib().df11_exponent_histogram(bad.data_ptr(), 16, hist.ctypes.data, None) == 9
