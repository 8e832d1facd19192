"""Selector artifact reader (host code in libveda; no GPU).

Files are written here byte by byte from the safetensors layout (8-byte
little-endian header length, JSON header, data section), so the reader is
checked against the format itself; conversions are checked bit for bit
against numpy's float16 and torch's bfloat16 / float8_e4m3fn casts.  The
published competition layout (100 float16 tensors of shape (56, 384, 128),
at most 560,000,000 bytes, metadata naming the hotkey) is exercised through
veda_selector_check with the same rules at a small size.
"""
import json
import struct

import numpy as np
import pytest
import torch

import learned_block_sparse_pool_b200 as veda
from learned_block_sparse_pool_b200 import binding as B


@pytest.fixture(scope="module", autouse=True)
def built():
    from learned_block_sparse_pool_b200 import build
    build.build()


def write_st(path, tensors, meta=None, header_override=None, pad_header=0, extra_data=b""):
    """tensors: list of (name, dtype string, shape, raw bytes) in data order."""
    header, data, off = {}, b"", 0
    for name, dt, shape, raw in tensors:
        header[name] = {"dtype": dt, "shape": list(shape), "data_offsets": [off, off + len(raw)]}
        data += raw
        off += len(raw)
    if meta is not None:
        header["__metadata__"] = meta
    hjson = header_override if header_override is not None else json.dumps(header)
    hb = hjson.encode() + b" " * pad_header
    path.write_bytes(struct.pack("<Q", len(hb)) + hb + data + extra_data)
    return path


def f16_tensor(name, shape, seed):
    a = np.random.default_rng(seed).standard_normal(shape).astype(np.float16)
    return (name, "F16", shape, a.tobytes()), a


def test_f16_read_as_fp32_and_bf16(tmp_path):
    t0, a0 = f16_tensor("layer0.q", (2, 8, 4), 0)
    t1, a1 = f16_tensor("layer0.k", (2, 8, 4), 1)
    p = write_st(tmp_path / "s.safetensors", [t0, t1], meta={"hotkey": "5Fabc"})
    with veda.Selector(str(p)) as s:
        assert len(s) == 2 and s.names() == ["layer0.q", "layer0.k"]
        assert s.info(0) == ("layer0.q", "F16", (2, 8, 4))
        assert s.metadata("hotkey") == "5Fabc" and s.metadata("nope") is None
        got32 = s.read("layer0.k", torch.float32)
        assert torch.equal(got32, torch.from_numpy(a1.astype(np.float32)))
        got16 = s.read("layer0.q", torch.bfloat16)
        want16 = torch.from_numpy(a0.astype(np.float32)).to(torch.bfloat16)
        assert torch.equal(got16.view(torch.int16), want16.view(torch.int16))
        s.check(2, (2, 8, 4), max_file_bytes=10_000, required_meta_key="hotkey")


def test_f16_special_values(tmp_path):
    vals = np.array([0.0, -0.0, 1.0, -2.5, 65504.0, 6.1e-5, 5.96e-8, -5.96e-8, np.inf, -np.inf, np.nan,
                     1e-6, 3.14159], np.float16)
    p = write_st(tmp_path / "s.safetensors", [("w", "F16", (13,), vals.tobytes())])
    with veda.Selector(str(p)) as s:
        got = s.read("w", torch.float32).numpy()
        want = vals.astype(np.float32)
        assert np.array_equal(np.isnan(got), np.isnan(want))
        m = ~np.isnan(want)
        assert np.array_equal(got[m].view(np.uint32), want[m].view(np.uint32))


def test_fp8_e4m3_every_code_with_scale(tmp_path):
    codes = np.arange(256, dtype=np.uint8)
    p = write_st(tmp_path / "s.safetensors", [("w", "F8_E4M3", (16, 16), codes.tobytes())])
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32).reshape(16, 16)
    with veda.Selector(str(p)) as s:
        got = s.read("w", torch.float32)
        assert torch.equal(torch.isnan(got), torch.isnan(want))
        m = ~torch.isnan(want)
        assert torch.equal(got[m], want[m])
        got_s = s.read("w", torch.bfloat16, scale=0.25)
        want_s = (want * 0.25).to(torch.bfloat16)
        assert torch.equal(got_s[m].float(), want_s[m].float())    # exact: e4m3 * 2^-2 fits bf16


def test_bf16_and_f32_stored(tmp_path):
    x = torch.randn(3, 5)
    p = write_st(tmp_path / "s.safetensors", [("a", "BF16", (3, 5), x.to(torch.bfloat16).view(torch.int16).numpy().tobytes()),
                                              ("b", "F32", (3, 5), x.numpy().tobytes())])
    with veda.Selector(str(p)) as s:
        assert torch.equal(s.read("a", torch.float32), x.to(torch.bfloat16).float())
        assert torch.equal(s.read("b", torch.float32), x)
        assert torch.equal(s.read("b", torch.bfloat16).view(torch.int16), x.to(torch.bfloat16).view(torch.int16))


def test_layout_check_rejections(tmp_path):
    t = [f16_tensor(f"l{i}.{qk}", (3, 4, 2), i * 2 + j)[0] for i in range(2) for j, qk in enumerate("qk")]
    p = write_st(tmp_path / "s.safetensors", t, meta={"hotkey": "x"})
    with veda.Selector(str(p)) as s:
        s.check(4, (3, 4, 2), 0, "hotkey")
        for args in [(5, (3, 4, 2), 0, None), (4, (3, 4, 3), 0, None), (4, (3, 4), 0, None),
                     (4, (3, 4, 2), 100, None), (4, (3, 4, 2), 0, "owner")]:
            with pytest.raises(B.VedaError) as e:
                s.check(*args)
            assert e.value.status == B.VEDA_ERR_FORMAT, args
        with pytest.raises(B.VedaError) as e:     # the competition layout: 100 x (56, 384, 128)
            s.check_published("hotkey")
        assert e.value.status == B.VEDA_ERR_FORMAT
    p32 = write_st(tmp_path / "f32.safetensors", [("w", "F32", (3, 4, 2), np.zeros(24, np.float32).tobytes())])
    with veda.Selector(str(p32)) as s:
        with pytest.raises(B.VedaError) as e:     # float32 is not a published selector dtype
            s.check(1, (3, 4, 2))
        assert e.value.status == B.VEDA_ERR_FORMAT


def _open_status(path):
    h = B.ctypes.c_void_p()
    st = B.lib().veda_selector_open(str(path).encode(), B.ctypes.byref(h))
    if st == 0:
        B.lib().veda_selector_close(h)
    return st


def test_malformed_files_rejected(tmp_path):
    raw = np.zeros(8, np.float16).tobytes()
    ok = [("w", "F16", (8,), raw)]
    good = write_st(tmp_path / "good.safetensors", ok)
    assert _open_status(good) == 0
    assert _open_status(write_st(tmp_path / "pad.safetensors", ok, pad_header=7)) == 0   # trailing spaces
    cases = {
        "gap": json.dumps({"w": {"dtype": "F16", "shape": [8], "data_offsets": [2, 18]}}),
        "overlap": json.dumps({"a": {"dtype": "F16", "shape": [4], "data_offsets": [0, 8]},
                               "b": {"dtype": "F16", "shape": [4], "data_offsets": [6, 14]}}),
        "past_end": json.dumps({"w": {"dtype": "F16", "shape": [16], "data_offsets": [0, 32]}}),
        "size_mismatch": json.dumps({"w": {"dtype": "F16", "shape": [7], "data_offsets": [0, 16]}}),
        "bad_dtype": json.dumps({"w": {"dtype": "F64", "shape": [2], "data_offsets": [0, 16]}}),
        "extra_field": json.dumps({"w": {"dtype": "F16", "shape": [8], "data_offsets": [0, 16], "x": 1}}),
        "negative_dim": json.dumps({"w": {"dtype": "F16", "shape": [-8], "data_offsets": [0, 16]}}),
        "float_offset": '{"w": {"dtype": "F16", "shape": [8], "data_offsets": [0, 16.0]}}',
        "duplicate": '{"w": {"dtype": "F16", "shape": [8], "data_offsets": [0, 16]}, '
                     '"w": {"dtype": "F16", "shape": [8], "data_offsets": [0, 16]}}',
        "truncated_json": '{"w": {"dtype": "F16", "shape": [8], "data_offsets": [0, 16]',
        "not_object": '[1, 2]',
        "metadata_number": json.dumps({"w": {"dtype": "F16", "shape": [8], "data_offsets": [0, 16]},
                                       "__metadata__": {"k": 3}}),
    }
    for name, hdr in cases.items():
        p = write_st(tmp_path / f"{name}.safetensors", ok, header_override=hdr)
        assert _open_status(p) == B.VEDA_ERR_FORMAT, name
    # trailing data past the last tensor, a header length beyond the file, a stub
    assert _open_status(write_st(tmp_path / "tail.safetensors", ok, extra_data=b"\0" * 4)) == B.VEDA_ERR_FORMAT
    big = tmp_path / "biglen.safetensors"
    big.write_bytes(struct.pack("<Q", 1 << 40) + b"{}")
    assert _open_status(big) == B.VEDA_ERR_FORMAT
    (tmp_path / "stub.safetensors").write_bytes(b"\x01\x02")
    assert _open_status(tmp_path / "stub.safetensors") == B.VEDA_ERR_FORMAT
    assert _open_status(tmp_path / "missing.safetensors") == B.VEDA_ERR_IO


def test_read_arguments_checked(tmp_path):
    p = write_st(tmp_path / "s.safetensors", [("w", "F16", (8,), np.ones(8, np.float16).tobytes())])
    with veda.Selector(str(p)) as s:
        L = B.lib()
        buf = (B.ctypes.c_float * 8)()
        assert L.veda_selector_read(s._h, 0, B.VEDA_F32, 1.0, buf, 8 * 4) == 0
        assert L.veda_selector_read(s._h, 0, B.VEDA_F32, 1.0, buf, 8 * 4 - 1) == B.VEDA_ERR_INVALID_ARG
        assert L.veda_selector_read(s._h, 1, B.VEDA_F32, 1.0, buf, 8 * 4) == B.VEDA_ERR_INVALID_ARG
        assert L.veda_selector_read(s._h, 0, 7, 1.0, buf, 8 * 4) == B.VEDA_ERR_INVALID_ARG
        assert L.veda_selector_read(s._h, 0, B.VEDA_F32, 0.0, buf, 8 * 4) == B.VEDA_ERR_INVALID_ARG
        assert list(buf) == [1.0] * 8
        with pytest.raises(B.VedaError):
            s.read("missing")
