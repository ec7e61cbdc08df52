"""DF11 tensors to and from a file.

The file has the safetensors layout:
- an 8-byte little-endian header length;
- a UTF-8 JSON header naming each stored buffer with its dtype, shape and byte range;
- the buffers back to back, with no holes.

Each compressed tensor `name` is stored as raw buffers:
- `name.bitstream`, `name.gaps`, `name.chunk_counts`, `name.code_lengths` and `name.sign_mantissa`
  (U8);
- `name.block_out_pos` and `name.luts` (U32).

Its format parameters, original shape and element order (rows interleaved per 16 columns; 1 for
row-major) go in the header's `__metadata__` as JSON under `name.df11`. The header is padded with spaces so that the data start at a 16-byte boundary.
Every buffer's length is a multiple of 16 (`block_out_pos` is zero-padded to one), so every buffer
of a file starts 16-byte aligned, ready to be mapped.

The pages describe saving a compressed model as its compressed weights plus the Huffman tables
("DFloat11无损压缩技术：基于哈夫曼编码的BFloat16大模型显存优化方案" §5.2); this layout is this
library's own.
"""
from __future__ import annotations

import json
import os
import struct
from typing import Dict, Mapping, Optional

import numpy as np

from . import Df11Host, Params

_FORMAT = "df11"
_VERSION = "1"
# (suffix, dtype name, numpy dtype) in storage order
_BUFFERS = (
    ("bitstream", "U8", np.uint8),
    ("gaps", "U8", np.uint8),
    ("chunk_counts", "U8", np.uint8),
    ("sign_mantissa", "U8", np.uint8),
    ("luts", "U32", np.uint32),
    ("code_lengths", "U8", np.uint8),
    ("block_out_pos", "U32", np.uint32),
)
_PARAM_FIELDS = [f for f, _ in Params._fields_]


def _expected_sizes(p: Params) -> Dict[str, int]:
    """Element counts of each buffer as the builder writes them."""
    C, T, nb = int(p.chunk_bytes), int(p.threads_per_block), int(p.num_blocks)
    return {
        "bitstream": nb * T * C + 16,
        "gaps": nb * T * 5 // 8 + 16,
        "chunk_counts": nb * T + 16,
        "sign_mantissa": (int(p.n) + 15) // 16 * 16,
        "luts": int(p.num_luts) * 256,
        "code_lengths": 256,
        "block_out_pos": nb + 1,
    }


def save(path: str, tensors: Mapping[str, Df11Host],
         metadata: Optional[Mapping[str, str]] = None) -> None:
    """Write compressed tensors (host form) to `path`."""
    header: Dict[str, object] = {}
    meta = {"format": _FORMAT, "version": _VERSION}
    if metadata:
        for k, v in metadata.items():
            if not isinstance(v, str):
                raise TypeError("metadata values must be strings")
            meta[k] = v
    blobs = []
    offset = 0
    for name, h in tensors.items():
        params = {f: int(getattr(h.params, f)) for f in _PARAM_FIELDS}
        meta[f"{name}.df11"] = json.dumps({"params": params, "shape": list(h.shape),
                                           "interleave": int(getattr(h, "interleave", 1))})
        for suffix, dname, dt in _BUFFERS:
            a = np.ascontiguousarray(getattr(h, suffix), dtype=dt)
            if suffix == "block_out_pos" and a.nbytes % 16:
                a = np.concatenate([a, np.zeros((16 - a.nbytes % 16) // 4, dt)])
            header[f"{name}.{suffix}"] = {"dtype": dname, "shape": [int(a.size)],
                                          "data_offsets": [offset, offset + a.nbytes]}
            blobs.append(a)
            offset += a.nbytes
    header["__metadata__"] = meta
    text = json.dumps(header, separators=(",", ":")).encode()
    text += b" " * ((-(8 + len(text))) % 16)
    tmp = path + ".tmp"
    with open(tmp, "wb") as f:
        f.write(struct.pack("<Q", len(text)))
        f.write(text)
        for a in blobs:
            f.write(a.tobytes())
    os.replace(tmp, path)


def _read_header(f, file_size: int):
    raw = f.read(8)
    if len(raw) != 8:
        raise ValueError("not a DF11 file: shorter than its header length")
    (hlen,) = struct.unpack("<Q", raw)
    if hlen > file_size - 8:
        raise ValueError("header length runs past the end of the file")
    try:
        header = json.loads(f.read(hlen).decode())
    except (UnicodeDecodeError, json.JSONDecodeError) as e:
        raise ValueError(f"header is not JSON: {e}") from None
    meta = header.pop("__metadata__", {})
    if meta.get("format") != _FORMAT:
        raise ValueError("not a DF11 file (no df11 format tag in the metadata)")
    if meta.get("version") != _VERSION:
        raise ValueError(f"unsupported DF11 file version {meta.get('version')!r}")
    return 8 + hlen, header, meta


def load(path: str) -> Dict[str, Df11Host]:
    """Read every compressed tensor of `path` (host form).  Raises
    ValueError when the file is not a consistent DF11 file."""
    size = os.path.getsize(path)
    with open(path, "rb") as f:
        start, header, meta = _read_header(f, size)
        data_size = size - start
        # the buffers must tile the data section exactly (no holes, no overlap)
        spans = sorted((tuple(v["data_offsets"]), k) for k, v in header.items())
        pos = 0
        for (b, e), k in spans:
            if b != pos or e < b:
                raise ValueError(f"buffer {k!r} does not continue the data section")
            pos = e
        if pos != data_size:
            raise ValueError("buffers do not cover the data section exactly")
        out: Dict[str, Df11Host] = {}
        names = [k[: -len(".df11")] for k in meta if k.endswith(".df11")]
        for name in names:
            info = json.loads(meta[f"{name}.df11"])
            p = Params(**{k: int(v) for k, v in info["params"].items() if k in _PARAM_FIELDS})
            want = _expected_sizes(p)
            arrays = {}
            for suffix, dname, dt in _BUFFERS:
                entry = header.get(f"{name}.{suffix}")
                if entry is None:
                    raise ValueError(f"{name}: buffer {suffix} missing")
                if entry["dtype"] != dname:
                    raise ValueError(f"{name}.{suffix}: dtype {entry['dtype']}, expected {dname}")
                b, e = entry["data_offsets"]
                count = (e - b) // np.dtype(dt).itemsize
                if count * np.dtype(dt).itemsize != e - b or entry["shape"] != [count]:
                    raise ValueError(f"{name}.{suffix}: shape and byte range disagree")
                need = want[suffix]
                if count < need or (suffix != "block_out_pos" and count != need):
                    raise ValueError(f"{name}.{suffix}: {count} elements, the parameters "
                                     f"say {need}")
                f.seek(start + b)
                a = np.frombuffer(f.read(e - b), dtype=dt)
                arrays[suffix] = a[:need].copy()
            out[name] = Df11Host(params=p, shape=tuple(info["shape"]),
                                 interleave=int(info.get("interleave", 1)), **arrays)
        return out
