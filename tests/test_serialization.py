"""DF11 files (huffman_decode_df11_b200.serialization): the safetensors
layout, exact round trips, and rejection of inconsistent files.  CPU only."""
import json
import os
import struct

import numpy as np
import pytest

import workloads
import huffman_decode_df11_b200 as df11
from huffman_decode_df11_b200 import serialization as ser

FIELDS = [f for f, _ in df11.Params._fields_]


def _tensors():
    rng = np.random.default_rng(0)
    a = df11.compress(workloads.gaussian_bf16(200_003, 0.02, 1).view(-1, 200_003), 8, 256)
    b = df11.compress(workloads.adversarial_mix(1 << 16, 2).view(256, 256), 24, 256)
    c = df11.compress(rng.integers(0, 1 << 16, 5000).astype(np.uint16), 16, 128)
    e = df11.compress(np.zeros(0, np.uint16))
    return {"layers.0.q_proj": a, "adversarial": b, "patterns": c, "empty": e}


def _same(h, g):
    assert [getattr(h.params, f) for f in FIELDS] == [getattr(g.params, f) for f in FIELDS]
    assert tuple(h.shape) == tuple(g.shape)
    for k in ("bitstream", "gaps", "chunk_counts", "sign_mantissa", "luts", "code_lengths",
              "block_out_pos"):
        assert np.array_equal(getattr(h, k), getattr(g, k)), k


def test_round_trip_is_exact(tmp_path):
    ts = _tensors()
    path = str(tmp_path / "w.df11")
    ser.save(path, ts, metadata={"model": "synthetic"})
    back = ser.load(path)
    assert set(back) == set(ts)
    for k in ts:
        _same(ts[k], back[k])


def test_file_has_the_safetensors_layout(tmp_path):
    """Parsed here from the layout's definition, independently of the
    reader: header length, JSON header, buffers tiling the data section
    with no holes, and 16-byte aligned buffer starts."""
    ts = _tensors()
    path = str(tmp_path / "w.df11")
    ser.save(path, ts)
    raw = open(path, "rb").read()
    (hlen,) = struct.unpack("<Q", raw[:8])
    header = json.loads(raw[8:8 + hlen])
    meta = header.pop("__metadata__")
    assert meta["format"] == "df11"
    data = raw[8 + hlen:]
    assert (8 + hlen) % 16 == 0
    spans = sorted(v["data_offsets"] for v in header.values())
    assert spans[0][0] == 0 and spans[-1][1] == len(data)
    for (b0, e0), (b1, _) in zip(spans, spans[1:]):
        assert e0 == b1
    for v in header.values():
        b, e = v["data_offsets"]
        assert b % 16 == 0
        size = {"U8": 1, "U32": 4}[v["dtype"]]
        assert v["shape"] == [(e - b) // size]
    # a buffer read straight from its byte range is the stored array
    h = ts["layers.0.q_proj"]
    b, e = header["layers.0.q_proj.bitstream"]["data_offsets"]
    assert np.array_equal(np.frombuffer(data[b:e], np.uint8), h.bitstream)


def test_inconsistent_files_are_rejected(tmp_path):
    ts = {"w": _tensors()["layers.0.q_proj"]}
    path = str(tmp_path / "w.df11")
    ser.save(path, ts)
    raw = bytearray(open(path, "rb").read())
    (hlen,) = struct.unpack("<Q", raw[:8])
    header = json.loads(raw[8:8 + hlen])

    def write(h, data=None):
        text = json.dumps(h).encode()
        text += b" " * ((-(8 + len(text))) % 16)
        p = str(tmp_path / "bad.df11")
        with open(p, "wb") as f:
            f.write(struct.pack("<Q", len(text)) + text + (raw[8 + hlen:] if data is None else data))
        return p

    with pytest.raises(ValueError):  # truncated data section
        ser.load(write(header, raw[8 + hlen:-16]))
    h = json.loads(json.dumps(header))
    h["w.gaps"]["data_offsets"][1] += 16           # overlap / hole
    with pytest.raises(ValueError):
        ser.load(write(h))
    h = json.loads(json.dumps(header))
    info = json.loads(h["__metadata__"]["w.df11"])
    info["params"]["num_blocks"] += 1                # parameters disagree with the buffers
    h["__metadata__"]["w.df11"] = json.dumps(info)
    with pytest.raises(ValueError):
        ser.load(write(h))
    h = json.loads(json.dumps(header))
    h["__metadata__"]["format"] = "other"
    with pytest.raises(ValueError):
        ser.load(write(h))
    p = str(tmp_path / "short.df11")
    open(p, "wb").write(b"\x01\x02")
    with pytest.raises(ValueError):
        ser.load(p)
    assert not os.path.exists(path + ".tmp")


def test_loaded_tensors_decode_like_the_originals(tmp_path):
    """The oracle decodes a loaded tensor back to the original words."""
    import oracle
    w = workloads.as_numpy_u16(workloads.adversarial_mix(1 << 15, 9))
    path = str(tmp_path / "w.df11")
    ser.save(path, {"w": df11.compress(w)})
    h = ser.load(path)["w"]
    out, end, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa, h.n)
    assert end == h.params.total_bits
    assert np.array_equal(out, w)


def test_interleave_survives_a_round_trip(tmp_path):
    w = np.arange(64 * 32, dtype=np.uint16).reshape(64, 32) % 977
    h = df11.compress(w, 8, 128, interleave=8)
    path = str(tmp_path / "i.df11")
    ser.save(path, {"w": h})
    back = ser.load(path)["w"]
    assert back.interleave == 8 and back.shape == (64, 32)
    assert np.array_equal(back.bitstream, h.bitstream)
