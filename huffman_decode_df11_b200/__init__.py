"""DF11 (DFloat11) lossless BF16 weight decode on B200 (sm_100a).

Thin Python binding over ``libdf11.so`` (built from ``csrc/``; C ABI declared
in ``include/df11.h``).  This module only marshals arguments: every step of
the decode runs in the library's CUDA kernel, and the format builder runs in
the library's host C++ code.  There is no fallback: if the library cannot be
loaded, importing the binding's entry points raises.

PyTorch is used for device memory and streams only.

    >>> h = compress(bf16_weight)            # host, once ("compression")
    >>> d = to_device(h, "cuda")             # compressed tensors in HBM
    >>> w = decode(d)                        # BF16 in HBM, bit-identical
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

from . import _build

_PKG = os.path.dirname(os.path.abspath(__file__))

# ---------------------------------------------------------------------------
# ctypes mirror of include/df11.h

DF11_MAX_BATCH = 16
DF11_DECODE_TABLE_BYTES = 17664
STATUS = {
    0: "DF11_OK", 1: "DF11_ERR_NULL", 2: "DF11_ERR_ALIGN", 3: "DF11_ERR_FORMAT",
    4: "DF11_ERR_UNSUPPORTED", 5: "DF11_ERR_CUDA", 6: "DF11_ERR_TOO_LARGE",
    7: "DF11_ERR_INVALID", 8: "DF11_ERR_NOMEM", 9: "DF11_ERR_DEVICE",
}
DEV_ERRORS = {
    0: "DF11_DEV_OK", 1: "DF11_DEV_ERR_COUNT", 2: "DF11_DEV_ERR_OVERRUN",
    3: "DF11_DEV_ERR_TABLE", 4: "DF11_DEV_ERR_TIMEOUT", 5: "DF11_DEV_ERR_CAPACITY",
}


class Params(ctypes.Structure):
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
    ]


class TensorDesc(ctypes.Structure):
    _fields_ = [
        ("bitstream", ctypes.c_void_p),
        ("gaps", ctypes.c_void_p),
        ("chunk_counts", ctypes.c_void_p),
        ("block_out_pos", ctypes.c_void_p),
        ("luts", ctypes.c_void_p),
        ("code_lengths", ctypes.c_void_p),
        ("sign_mantissa", ctypes.c_void_p),
        ("out_bf16", ctypes.c_void_p),
        ("decode_table", ctypes.c_void_p),
        ("params", Params),
    ]


class GemvOp(ctypes.Structure):
    """df11_gemv: the matrix-vector product applied to one decoded tensor."""
    _fields_ = [("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("cols", ctypes.c_uint32),
                ("batch", ctypes.c_uint32), ("x_stride", ctypes.c_uint32),
                ("y_stride", ctypes.c_uint32), ("accumulate", ctypes.c_int32),
                ("interleave", ctypes.c_uint32)]


class HostTensor(ctypes.Structure):
    _fields_ = [
        ("params", Params),
        ("code_lengths", ctypes.c_uint8 * 256),
        ("bitstream", ctypes.POINTER(ctypes.c_uint8)),
        ("bitstream_bytes", ctypes.c_uint64),
        ("gaps", ctypes.POINTER(ctypes.c_uint8)),
        ("gaps_bytes", ctypes.c_uint64),
        ("block_out_pos", ctypes.POINTER(ctypes.c_uint32)),
        ("luts", ctypes.POINTER(ctypes.c_uint32)),
        ("sign_mantissa", ctypes.POINTER(ctypes.c_uint8)),
        ("sign_mantissa_bytes", ctypes.c_uint64),
        ("chunk_counts", ctypes.POINTER(ctypes.c_uint8)),
        ("chunk_counts_bytes", ctypes.c_uint64),
    ]


class Df11Error(RuntimeError):
    pass


_lib = None


def lib():
    """The loaded libdf11.so (built in-tree on first use if stale or missing)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if _build._stale() and os.path.exists(_build.NVCC):
        path = _build.build()
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing and nvcc is not available to build it; the DF11 "
            "decode path has no CPU fallback")
    L = ctypes.CDLL(path)
    vp, u64, u32, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int32
    L.df11_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, u64, ctypes.POINTER(Params), vp, vp]
    L.df11_decode.restype = ctypes.c_int
    L.df11_decode_batched.argtypes = [ctypes.POINTER(TensorDesc), ctypes.c_int, vp, vp]
    L.df11_decode_batched.restype = ctypes.c_int
    L.df11_shared_bytes.argtypes = [ctypes.POINTER(Params)]
    L.df11_shared_bytes.restype = ctypes.c_size_t
    L.df11_supported.argtypes = [u32, u32]
    L.df11_supported.restype = ctypes.c_int
    L.df11_status_string.argtypes = [ctypes.c_int]
    L.df11_status_string.restype = ctypes.c_char_p
    L.df11_device_error_string.argtypes = [i32]
    L.df11_device_error_string.restype = ctypes.c_char_p
    L.df11_build.argtypes = [vp, u64, u32, u32, ctypes.c_int, ctypes.POINTER(HostTensor)]
    L.df11_build.restype = ctypes.c_int
    L.df11_host_tensor_free.argtypes = [ctypes.POINTER(HostTensor)]
    L.df11_build_decode_table.argtypes = [vp, vp, u32, vp, vp]
    L.df11_build_decode_table.restype = ctypes.c_int
    L.df11_gpu_build_begin.argtypes = [vp, u64, u32, u32, vp, ctypes.POINTER(Params), vp,
                                       ctypes.POINTER(vp)]
    L.df11_gpu_build_begin.restype = ctypes.c_int
    L.df11_gpu_build_finish.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        ctypes.POINTER(Params), vp]
    L.df11_gpu_build_finish.restype = ctypes.c_int
    L.df11_gpu_build_begin_batched.argtypes = [vp, vp, ctypes.c_int, u32, u32, vp, vp, vp, vp]
    L.df11_gpu_build_begin_batched.restype = ctypes.c_int
    L.df11_gpu_build_finish_batched.argtypes = [vp, ctypes.c_int, vp, vp, vp, vp]
    L.df11_gpu_build_finish_batched.restype = ctypes.c_int
    L.df11_gpu_build_layout.argtypes = [vp, ctypes.c_int, vp, vp]
    L.df11_gpu_build_layout.restype = u64
    L.df11_gpu_build_free.argtypes = [vp]
    L.df11_gpu_build_free.restype = None
    L.df11_decode_gemv.argtypes = [ctypes.POINTER(TensorDesc), ctypes.POINTER(GemvOp),
                                   ctypes.c_int, vp, vp]
    L.df11_decode_gemv.restype = ctypes.c_int
    L.df11_decode_gemm.argtypes = [ctypes.POINTER(TensorDesc), ctypes.POINTER(GemvOp),
                                   ctypes.c_int, vp, vp]
    L.df11_decode_gemm.restype = ctypes.c_int
    L.df11_exponent_histogram.argtypes = [vp, u64, vp, vp]
    L.df11_exponent_histogram.restype = ctypes.c_int
    L.df11_test_withhold_copies.argtypes = [ctypes.c_int, u32]
    L.df11_test_withhold_copies.restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int, what: str):
    if status != 0:
        msg = lib().df11_status_string(status).decode()
        raise Df11Error(f"{what}: {STATUS.get(status, status)} ({msg})")


def supported(chunk_bytes: int, threads_per_block: int) -> bool:
    return bool(lib().df11_supported(chunk_bytes, threads_per_block))


# ---------------------------------------------------------------------------
# host side: the format builder

@dataclass
class Df11Host:
    """One compressed tensor in host memory (numpy arrays)."""
    params: Params
    code_lengths: np.ndarray   # uint8[256]
    bitstream: np.ndarray      # uint8
    gaps: np.ndarray           # uint8 (5-bit fields)
    block_out_pos: np.ndarray  # uint32[num_blocks + 1]
    luts: np.ndarray           # uint32[num_luts * 256]
    sign_mantissa: np.ndarray  # uint8 (n rounded up to 16)
    chunk_counts: np.ndarray   # uint8, codewords starting in each chunk
    shape: tuple = ()
    interleave: int = 1        # rows interleaved per 16 columns in the stream (1: row-major)

    @property
    def n(self) -> int:
        return int(self.params.n)

    def compressed_bytes(self) -> int:
        """Bytes stored: bitstream + gaps + positions + tables + code lengths
        + sign/mantissa + chunk counts."""
        return (self.bitstream.nbytes + self.gaps.nbytes + self.block_out_pos.nbytes
                + self.luts.nbytes + 256 + self.sign_mantissa.nbytes
                + self.chunk_counts.nbytes)


def _as_u16_numpy(w) -> np.ndarray:
    if isinstance(w, torch.Tensor):
        t = w.detach()
        if t.dtype in (torch.bfloat16, torch.float16, torch.uint16):
            t = t.view(torch.int16)
        if t.dtype != torch.int16:
            raise TypeError("expected a 2-byte tensor of BF16 bit patterns")
        return t.cpu().contiguous().reshape(-1).numpy().view(np.uint16)
    a = np.ascontiguousarray(w).reshape(-1)
    if a.dtype.itemsize != 2:
        raise TypeError("expected 2-byte BF16 bit patterns")
    return a.view(np.uint16)


def _np_copy(ptr, count, dtype):
    if count == 0:
        return np.zeros(0, dtype)
    ctype = np.ctypeslib.as_ctypes_type(dtype)
    buf = ctypes.cast(ptr, ctypes.POINTER(ctype * count)).contents
    return np.frombuffer(buf, dtype=dtype, count=count).copy()


def interleave_rows(w, rows_per_block: int):
    """The element order df11_gemv calls R rows interleaved (R =
    rows_per_block, a power of two up to 128): for each block of R rows and
    each group of 16 columns, the R rows' 16 elements one after another.
    R = 128 makes every 2048 elements one 128 x 16 tile of the tensor-core
    product (decode_gemm).  Takes a 2-D array or tensor (rows a multiple of
    R, columns of 16) and returns it flattened in that order."""
    R = int(rows_per_block)
    rows, cols = w.shape
    if R < 1 or R > 128 or R & (R - 1) or rows % R or cols % 16:
        raise ValueError(f"cannot interleave a {rows}x{cols} matrix by {R} rows")
    v = w.reshape(rows // R, R, cols // 16, 16)
    v = v.permute(0, 2, 1, 3) if isinstance(v, torch.Tensor) else v.transpose(0, 2, 1, 3)
    return v.reshape(-1) if isinstance(v, torch.Tensor) else np.ascontiguousarray(v).reshape(-1)


def deinterleave_rows(flat, shape, rows_per_block: int):
    """The inverse of interleave_rows: a stream-ordered flat array or
    tensor back to the rows x cols matrix."""
    R = int(rows_per_block)
    rows, cols = shape
    v = flat.reshape(rows // R, cols // 16, R, 16)
    v = v.permute(0, 2, 1, 3) if isinstance(v, torch.Tensor) else v.transpose(0, 2, 1, 3)
    return v.reshape(rows, cols)


def compress(w, chunk_bytes: int = 24, threads_per_block: int = 256,
             threads: int = 0, interleave: int = 1) -> Df11Host:
    """Encode a BF16 tensor (host or device; copied to host) into DF11.
    The default chunk of 24 bitstream bytes per thread decodes fastest on
    B200 of the built kernel shapes (fewer per-chunk setup steps per element
    than 8 or 16) and stores less metadata; any multiple of 4 from 4 to 28 is
    a valid format."""
    shape = tuple(w.shape) if hasattr(w, "shape") else ()
    a = _as_u16_numpy(w)
    if interleave != 1:
        a = interleave_rows(a.reshape(shape), interleave)
    h = HostTensor()
    L = lib()
    _check(L.df11_build(a.ctypes.data if a.size else None, a.size, chunk_bytes,
                        threads_per_block, threads, ctypes.byref(h)), "df11_build")
    try:
        p = Params.from_buffer_copy(h.params)
        out = Df11Host(
            params=p,
            code_lengths=np.frombuffer(bytes(h.code_lengths), np.uint8).copy(),
            bitstream=_np_copy(h.bitstream, h.bitstream_bytes, np.uint8),
            gaps=_np_copy(h.gaps, h.gaps_bytes, np.uint8),
            block_out_pos=_np_copy(h.block_out_pos, p.num_blocks + 1, np.uint32),
            luts=_np_copy(h.luts, p.num_luts * 256, np.uint32),
            sign_mantissa=_np_copy(h.sign_mantissa, h.sign_mantissa_bytes, np.uint8),
            chunk_counts=_np_copy(h.chunk_counts, h.chunk_counts_bytes, np.uint8),
            shape=shape,
            interleave=int(interleave),
        )
    finally:
        L.df11_host_tensor_free(ctypes.byref(h))
    return out


# ---------------------------------------------------------------------------
# device side

@dataclass
class Df11Device:
    """One compressed tensor resident in device memory (torch tensors)."""
    params: Params
    bitstream: torch.Tensor
    gaps: torch.Tensor
    block_out_pos: torch.Tensor
    luts: torch.Tensor
    code_lengths: torch.Tensor
    sign_mantissa: torch.Tensor
    chunk_counts: Optional[torch.Tensor] = None
    shape: tuple = ()
    decode_table: Optional[torch.Tensor] = None  # df11_build_decode_table output
    interleave: int = 1  # rows interleaved per 16 columns in the stream (1: row-major)

    @classmethod
    def _in_block(cls, params: Params, block: torch.Tensor, offs: tuple, sizes: tuple,
                  shape: tuple, interleave: int) -> "Df11Device":
        """A tensor whose buffers are byte ranges of one device allocation
        (offsets and sizes in the order of _BUFFERS).  The tensor view of a
        buffer is made when the buffer is first used; pointers for a decode
        come straight from the allocation."""
        d = cls.__new__(cls)
        d.__dict__.update(params=params, shape=shape, interleave=interleave, decode_table=None,
                          _block=block, _offs=offs, _sizes=sizes)
        return d

    def __getattr__(self, name):
        # only reached for a buffer of a _in_block tensor not yet viewed
        dd = self.__dict__
        i = _BUFFER_INDEX.get(name)
        if i is None or "_offs" not in dd:
            raise AttributeError(name)
        off = dd["_offs"][i]
        v = dd["_block"][off:off + dd["_sizes"][i]]
        if _BUFFERS[i][1] is not None:
            v = v.view(_BUFFERS[i][1])
        dd[name] = v
        return v

    def _ptr(self, name: str) -> int:
        dd = self.__dict__
        if "_offs" in dd and name not in dd:
            return dd["_block"].data_ptr() + dd["_offs"][_BUFFER_INDEX[name]]
        return getattr(self, name).data_ptr()

    @property
    def n(self) -> int:
        return int(self.params.n)

    @property
    def device(self):
        b = self.__dict__.get("_block")
        return b.device if b is not None else self.bitstream.device

    def compressed_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.bitstream, self.gaps, self.block_out_pos, self.luts,
                    self.code_lengths, self.sign_mantissa)
                   + ((self.chunk_counts,) if self.chunk_counts is not None else ()))

    def desc(self, out: torch.Tensor, counts: bool = True) -> TensorDesc:
        cc = (self._ptr("chunk_counts") if counts and ("_offs" in self.__dict__
                                                        or self.chunk_counts is not None)
              else None)
        dt = self.decode_table.data_ptr() if self.decode_table is not None else None
        p = self._ptr
        return TensorDesc(p("bitstream"), p("gaps"), cc, p("block_out_pos"), p("luts"),
                          p("code_lengths"), p("sign_mantissa"), out.data_ptr(), dt, self.params)


# the buffers of a device tensor in the order of df11_gpu_build_out, with the
# view each gets (None: bytes)
_BUFFERS = (("bitstream", None), ("gaps", None), ("chunk_counts", None),
            ("block_out_pos", torch.int32), ("luts", torch.int32), ("code_lengths", None),
            ("sign_mantissa", None))
_BUFFER_INDEX = {name: i for i, (name, _) in enumerate(_BUFFERS)}
# a tensor built by _in_block has no chunk_counts attribute until first use;
# the default stays in the constructor
del Df11Device.chunk_counts


def _np_to(t: np.ndarray, device, pin: bool = False) -> torch.Tensor:
    x = torch.from_numpy(t)
    if pin:
        x = x.pin_memory()
    return x.to(device, non_blocking=pin)


def to_device(h: Df11Host, device="cuda", decode_table: bool = True) -> Df11Device:
    """Copy a compressed tensor into device memory (16-byte aligned buffers)
    and, unless decode_table=False, derive its decode table there once
    (df11_build_decode_table) so that decode calls need not."""
    d = Df11Device(
        params=Params.from_buffer_copy(h.params),
        bitstream=_np_to(h.bitstream, device),
        gaps=_np_to(h.gaps, device),
        block_out_pos=_np_to(h.block_out_pos.view(np.int32), device),
        luts=_np_to(h.luts.view(np.int32), device),
        code_lengths=_np_to(h.code_lengths, device),
        sign_mantissa=_np_to(h.sign_mantissa, device),
        chunk_counts=_np_to(h.chunk_counts, device),
        shape=h.shape,
        interleave=int(getattr(h, "interleave", 1)),
    )
    if decode_table:
        d.decode_table = build_decode_table(d)
    return d


def to_host(d: Df11Device) -> Df11Host:
    """Copy a compressed tensor from device memory back into host arrays
    (the inverse of to_device; e.g. to save a tensor built on the device).
    Synchronises with the copies."""
    def arr(t, dtype):
        return t.cpu().numpy().view(dtype).copy()
    cc = d.chunk_counts
    return Df11Host(params=Params.from_buffer_copy(d.params),
                    code_lengths=arr(d.code_lengths, np.uint8),
                    bitstream=arr(d.bitstream, np.uint8), gaps=arr(d.gaps, np.uint8),
                    block_out_pos=arr(d.block_out_pos, np.uint32),
                    luts=arr(d.luts, np.uint32),
                    sign_mantissa=arr(d.sign_mantissa, np.uint8),
                    chunk_counts=arr(cc, np.uint8) if cc is not None else np.zeros(0, np.uint8),
                    shape=d.shape, interleave=int(getattr(d, "interleave", 1)))


class GpuBuildOut(ctypes.Structure):
    """df11_gpu_build_out: one tensor's phase-2 output buffers."""
    _fields_ = [(f, ctypes.c_void_p) for f in ("bitstream", "gaps", "chunk_counts",
                                               "block_out_pos", "luts", "code_lengths",
                                               "sign_mantissa")]


def compress_on_device(w: torch.Tensor, chunk_bytes: int = 24, threads_per_block: int = 256,
                       stream=None, decode_table: bool = True,
                       interleave: int = 1) -> Df11Device:
    """Encode a BF16 tensor that is in device memory into DF11 on the device
    (df11_gpu_build_begin / df11_gpu_build_finish): the same bytes and
    parameters as compress() of the same words, written straight into
    device buffers.  Synchronises the stream."""
    return compress_on_device_batched([w], chunk_bytes, threads_per_block, stream,
                                      decode_table, interleave)[0]


def compress_on_device_batched(ws: Sequence[torch.Tensor], chunk_bytes: int = 24,
                               threads_per_block: int = 256, stream=None,
                               decode_table: bool = True,
                               interleave: int = 1) -> List[Df11Device]:
    """compress_on_device for several tensors, with one stream
    synchronisation per phase for all of them
    (df11_gpu_build_begin_batched / _finish_batched)."""
    if len(ws) == 0:
        return []
    with torch.cuda.device(ws[0].device):
        return _compress_on_device_batched(ws, chunk_bytes, threads_per_block, stream,
                                           decode_table, interleave)


def _compress_on_device_batched(ws, chunk_bytes, threads_per_block, stream, decode_table,
                                interleave):
    count = len(ws)
    # the words as flat contiguous tensors (the interleaved copy, or the
    # tensor itself: only its address and size go to the library)
    flats, shapes = [], []
    dev = ws[0].get_device()
    for w in ws:
        if not w.is_cuda:
            raise ValueError("compress_on_device takes CUDA tensors; use compress() for host data")
        if w.dtype not in _WORD_DTYPES:
            raise TypeError(f"expected BF16 words (bfloat16, int16 or uint16), got {w.dtype}")
        if w.get_device() != dev:
            raise ValueError("all tensors of one batched build must be on one device")
        shapes.append(tuple(w.shape))
        if interleave != 1:
            flats.append(interleave_rows(w, interleave).contiguous())
        else:
            flats.append(w if w.is_contiguous() else w.contiguous())
    L = lib()
    sh = _stream_handle(stream)
    vp = ctypes.c_void_p
    nums = [f.numel() for f in flats]
    ptrs = (vp * count)(*[f.data_ptr() if k else None for f, k in zip(flats, nums)])
    ns = (ctypes.c_uint64 * count)(*nums)
    params = (Params * count)()
    lens = (ctypes.c_uint8 * (256 * count))()
    handles = (vp * count)()
    _check(L.df11_gpu_build_begin_batched(ptrs, ns, count, chunk_bytes, threads_per_block, sh,
                                          params, ctypes.cast(lens, vp), handles),
           "df11_gpu_build_begin_batched")
    try:
        # every output buffer of the call in one allocation (df11_gpu_build_layout)
        offs = (ctypes.c_uint64 * (7 * count))()
        sizes = (ctypes.c_uint64 * (7 * count))()
        total = L.df11_gpu_build_layout(params, count, offs, sizes)
        block = torch.empty(max(total, 256), dtype=torch.uint8, device=flats[0].device)
        addr = np.frombuffer(offs, dtype=np.uint64) + np.uint64(block.data_ptr())
        outs = (vp * (7 * count)).from_buffer(addr)
    except BaseException:
        for hnd in handles:
            L.df11_gpu_build_free(hnd)
        raise
    _check(L.df11_gpu_build_finish_batched(handles, count, ptrs, outs, params, sh),
           "df11_gpu_build_finish_batched")
    out = []
    il = int(interleave)
    for i, shape in enumerate(shapes):
        d = Df11Device._in_block(params[i], block, offs[7 * i:7 * i + 7],
                                 sizes[7 * i:7 * i + 7], shape, il)
        if decode_table:
            d.decode_table = build_decode_table(d, stream)
        out.append(d)
    return out


def exponent_histogram(w: torch.Tensor, stream=None) -> np.ndarray:
    """Counts of the 256 exponent values of a contiguous BF16 tensor in
    device memory (df11_exponent_histogram: allocates no device memory, for
    callers that cannot; synchronises the stream)."""
    if not w.is_cuda:
        raise ValueError("exponent_histogram takes a CUDA tensor")
    if w.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected BF16 words (bfloat16, int16 or uint16), got {w.dtype}")
    if not w.is_contiguous():
        # a contiguous copy would be a device allocation, which this call avoids
        raise ValueError("exponent_histogram takes a contiguous tensor")
    n = w.numel()
    hist = np.zeros(256, dtype=np.uint64)
    with torch.cuda.device(w.device):
        _check(lib().df11_exponent_histogram(w.data_ptr() if n else None, n,
                                             hist.ctypes.data, _stream_handle(stream)),
               "df11_exponent_histogram")
    return hist


def build_decode_table(d: Df11Device, stream=None) -> torch.Tensor:
    """The decode table of a device tensor (df11_build_decode_table)."""
    t = torch.empty(DF11_DECODE_TABLE_BYTES, dtype=torch.uint8, device=d.device)
    with torch.cuda.device(d.device):
        _check(lib().df11_build_decode_table(d._ptr("luts"), d._ptr("code_lengths"),
                                             int(d.params.num_luts), t.data_ptr(),
                                             _stream_handle(stream)), "df11_build_decode_table")
    return t


_WORD_DTYPES = (torch.bfloat16, torch.int16, torch.uint16)


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def empty_output(d: Df11Device) -> torch.Tensor:
    return torch.empty(max(d.n, 1), dtype=torch.bfloat16, device=d.device)[: d.n]


def decode(d: Df11Device, out: Optional[torch.Tensor] = None,
           err: Optional[torch.Tensor] = None, stream=None,
           counts: bool = True) -> torch.Tensor:
    """Decode into `out` (a flat BF16/int16 device tensor of n elements,
    allocated if None).  Asynchronous on `stream` (default: current stream).
    `err` is an optional int32 device tensor the kernel writes error codes
    into (see check_device_error).  With counts (the default, when the tensor
    carries chunk counts) the one-pass decode is used; counts=False runs the
    format the pages describe through df11_decode (count by decoding)."""
    if out is None:
        out = empty_output(d)
    _check_out(d, out)
    if counts and d.chunk_counts is not None:
        return decode_batched([d], [out], err=err, stream=stream)[0]
    p = Params.from_buffer_copy(d.params)
    with torch.cuda.device(d.device):
        _check(lib().df11_decode(
            d.bitstream.data_ptr(), d.gaps.data_ptr(), d.block_out_pos.data_ptr(),
            d.luts.data_ptr(), d.code_lengths.data_ptr(), d.sign_mantissa.data_ptr(),
            out.data_ptr(), d.n, ctypes.byref(p),
            err.data_ptr() if err is not None else None, _stream_handle(stream)),
            "df11_decode")
    return out


def _check_out(d: Df11Device, out: torch.Tensor):
    if out.numel() != d.n or not out.is_contiguous() or out.element_size() != 2:
        raise ValueError("out must be a contiguous 2-byte tensor with n elements")


def decode_batched(ds: Sequence[Df11Device], outs: Sequence[torch.Tensor],
                   err: Optional[torch.Tensor] = None, stream=None,
                   counts: bool = True):
    """Decode several tensors with one launch per 16 tensors."""
    if len(ds) != len(outs):
        raise ValueError("one output per tensor")
    for d, o in zip(ds, outs):
        _check_out(d, o)
    if not ds:
        return outs
    arr = (TensorDesc * len(ds))(*[d.desc(o, counts) for d, o in zip(ds, outs)])
    with torch.cuda.device(_one_device(ds, outs)):
        _check(lib().df11_decode_batched(arr, len(ds),
                                         err.data_ptr() if err is not None else None,
                                         _stream_handle(stream)), "df11_decode_batched")
    return outs


def _one_device(ds, others=()):
    """The one CUDA device of a call's tensors (the library's kernels run on
    the current device and check that every buffer is its own)."""
    dev = ds[0].device
    for t in list(ds) + list(others):
        if t.device != dev:
            raise ValueError(f"tensors of one call on {dev} and {t.device}")
    return dev


class DecodePlan:
    """A decode of fixed compressed tensors into fixed outputs (one layer's
    weights into its scratch buffers, say), prepared once: the descriptor
    array is built here, and every run() is one library call (one launch per
    16 tensors), as a layer-by-layer decode loop wants."""

    def __init__(self, ds: Sequence[Df11Device], outs: Sequence[torch.Tensor],
                 counts: bool = True):
        if len(ds) != len(outs):
            raise ValueError("one output per tensor")
        for d, o in zip(ds, outs):
            _check_out(d, o)
        self._keep = (list(ds), list(outs))  # the buffers the descriptors point to
        self._n = len(ds)
        self._arr = (TensorDesc * max(self._n, 1))(*[d.desc(o, counts) for d, o in zip(ds, outs)])
        self._lib = lib()
        self._device = _one_device(ds, outs) if ds else None

    @property
    def outs(self):
        return self._keep[1]

    def run(self, err: Optional[torch.Tensor] = None, stream=None):
        if self._device is not None and torch.cuda.current_device() != self._device.index:
            with torch.cuda.device(self._device):
                return self.run(err, stream)
        _check(self._lib.df11_decode_batched(self._arr, self._n,
                                             err.data_ptr() if err is not None else None,
                                             _stream_handle(stream)), "df11_decode_batched")
        return self._keep[1]


def _gemv_op(d: "Df11Device", x: torch.Tensor, y: torch.Tensor, accumulate: bool) -> GemvOp:
    """Check one (tensor, activations, outputs) triple and describe it."""
    if len(d.shape) != 2:
        raise ValueError("decode_gemv needs a 2-D weight (rows x cols)")
    rows, cols = d.shape
    if x.dtype not in (torch.bfloat16, torch.int16) or y.dtype != torch.float32:
        raise TypeError("x must be BF16 and y float32")
    x2 = x if x.dim() == 2 else x.view(1, -1)
    y2 = y if y.dim() == 2 else y.view(1, -1)
    if x2.shape[1] != cols or y2.shape[1] != rows or x2.shape[0] != y2.shape[0]:
        raise ValueError(f"shapes: W {rows}x{cols}, x {tuple(x.shape)}, y {tuple(y.shape)}")
    if x2.stride(1) != 1 or y2.stride(1) != 1:
        raise ValueError("x and y rows must be contiguous")
    if x2.device != d.device or y2.device != d.device:
        raise ValueError("x and y must be on the weight's device")
    return GemvOp(x2.data_ptr(), y2.data_ptr(), cols, x2.shape[0], x2.stride(0),
                  y2.stride(0), 1 if accumulate else 0, int(getattr(d, "interleave", 1)))


def decode_gemv(ds: Sequence["Df11Device"], xs: Sequence[torch.Tensor],
                ys: Sequence[torch.Tensor], accumulate: bool = False,
                err: Optional[torch.Tensor] = None, stream=None):
    """y = W x (or y += W x) for each compressed weight W (rows x cols) with
    BF16 activations x (batch x cols, or cols) into float32 y (batch x
    rows, or rows), decoding W inside the product (df11_decode_gemv): the
    BF16 weights never reach memory.  One launch per 16 tensors."""
    if not (len(ds) == len(xs) == len(ys)):
        raise ValueError("one x and one y per tensor")
    n = len(ds)
    if n == 0:
        return
    descs = (TensorDesc * n)(*[d.desc(torch.empty(0, device=d.device)) for d in ds])
    for i, d in enumerate(ds):
        descs[i].out_bf16 = None
    ops = (GemvOp * n)(*[_gemv_op(d, x, y, accumulate) for d, x, y in zip(ds, xs, ys)])
    with torch.cuda.device(_one_device(ds)):
        _check(lib().df11_decode_gemv(descs, ops, n,
                                      err.data_ptr() if err is not None else None,
                                      _stream_handle(stream)), "df11_decode_gemv")


def decode_gemm(ds: Sequence["Df11Device"], xs: Sequence[torch.Tensor],
                ys: Sequence[torch.Tensor], accumulate: bool = False,
                err: Optional[torch.Tensor] = None, stream=None):
    """y = W x (or y += W x) on the tensor cores for weights W (rows x cols)
    compressed with interleave=128 (and chunk_bytes 8 or 16) and BF16
    activations x (batch x cols, batch 1..128) into float32 y (batch x
    rows), decoding W inside the product (df11_decode_gemm): the BF16
    weights never reach memory.  One launch for up to 16 weights."""
    if not (len(ds) == len(xs) == len(ys)):
        raise ValueError("one x and one y per tensor")
    n = len(ds)
    if n == 0:
        return
    if n > DF11_MAX_BATCH:
        raise ValueError(f"at most {DF11_MAX_BATCH} weights per call")
    for d in ds:
        if int(getattr(d, "interleave", 1)) != 128:
            raise ValueError("decode_gemm needs weights compressed with interleave=128")
    descs = (TensorDesc * n)(*[d.desc(torch.empty(0, device=d.device)) for d in ds])
    for i in range(n):
        descs[i].out_bf16 = None
    ops = (GemvOp * n)(*[_gemv_op(d, x, y, accumulate) for d, x, y in zip(ds, xs, ys)])
    with torch.cuda.device(_one_device(ds)):
        _check(lib().df11_decode_gemm(descs, ops, n,
                                      err.data_ptr() if err is not None else None,
                                      _stream_handle(stream)), "df11_decode_gemm")


def new_error_word(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_device_error(err: torch.Tensor):
    """Raise if the kernel flagged inconsistent data (synchronises)."""
    code = int(err.item())
    if code != 0:
        msg = lib().df11_device_error_string(code).decode()
        raise Df11Error(f"decode reported {DEV_ERRORS.get(code, code)}: {msg}")
