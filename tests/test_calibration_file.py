"""The Smooth-QK calibration file (hifa4_calibration_save / _load in the product library),
on CPU: a round trip keeps every bit of s, s_inv and alpha; the header is the documented
layout (checked field by field with struct, the checksum with zlib's CRC-32); a wrong
magic, a wrong version, a truncated or extended file and a flipped payload bit are all
refused with HIFA4_ERR_IO, and the caller's arrays are left untouched."""
import struct
import zlib

import numpy as np
import pytest
import torch

from bit_flashattention_b200 import hifa4


def _scales(Hkv=8, d=128, seed=5):
    import oracle
    from bit_flashattention_b200 import configs, gen
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2 * Hkv, Hkv=Hkv, N=256, d=d)
    qc, kc, _ = gen.inputs(w, calib=True)
    s, sinv = oracle.calibrate(qc, kc, 0.5)
    return torch.from_numpy(s), torch.from_numpy(sinv)


def test_round_trip_keeps_every_bit(tmp_path):
    s, sinv = _scales()
    p = tmp_path / "cal.bin"
    hifa4.hifa4_calibration_save(p, s, sinv, 0.5)
    s2, si2, a2 = hifa4.hifa4_calibration_load(p)
    assert torch.equal(s2.view(torch.int32), s.view(torch.int32))
    assert torch.equal(si2.view(torch.int32), sinv.view(torch.int32))
    assert a2 == 0.5


def test_file_layout(tmp_path):
    s, sinv = _scales(Hkv=2, d=64)
    p = tmp_path / "cal.bin"
    hifa4.hifa4_calibration_save(p, s, sinv, 0.25)
    raw = p.read_bytes()
    magic, ver, hk, dd, alpha, crc = struct.unpack("<8sIiifI", raw[:28])
    assert (magic, ver, hk, dd, alpha) == (b"HIFA4CAL", 1, 2, 64, 0.25)
    body = raw[28:]
    assert len(body) == 2 * 2 * 64 * 4
    assert crc == zlib.crc32(body)
    assert np.array_equal(np.frombuffer(body[:512], "<f4").reshape(2, 64), s.numpy())
    assert np.array_equal(np.frombuffer(body[512:], "<f4").reshape(2, 64), sinv.numpy())


@pytest.mark.parametrize("damage", ["magic", "version", "truncated", "extended", "payload"])
def test_damaged_files_are_refused(tmp_path, damage):
    s, sinv = _scales(Hkv=2, d=64)
    p = tmp_path / "cal.bin"
    hifa4.hifa4_calibration_save(p, s, sinv, 0.5)
    raw = bytearray(p.read_bytes())
    if damage == "magic":
        raw[0:8] = b"HIFA4CAX"
    elif damage == "version":
        raw[8:12] = struct.pack("<I", 2)
    elif damage == "truncated":
        raw = raw[:-4]
    elif damage == "extended":
        raw += b"\0"
    else:
        raw[100] ^= 0x01
    p.write_bytes(bytes(raw))
    with pytest.raises(hifa4.Hifa4Error) as e:
        hifa4.hifa4_calibration_load(p)
    assert e.value.code == hifa4.ERR_IO
    assert hifa4.status_string(hifa4.ERR_IO) == "HIFA4_ERR_IO"


def test_arguments_and_capacity(tmp_path):
    import ctypes
    L = hifa4.lib()
    s, sinv = _scales(Hkv=2, d=64)
    p = tmp_path / "cal.bin"
    with pytest.raises(hifa4.Hifa4Error):
        hifa4.hifa4_calibration_save(p, s, sinv, -1.0)
    with pytest.raises(hifa4.Hifa4Error):
        hifa4.hifa4_calibration_load(tmp_path / "missing.bin")
    hifa4.hifa4_calibration_save(p, s, sinv, 0.5)
    hk, dd, al = ctypes.c_int(), ctypes.c_int(), ctypes.c_float()
    small = np.full(10, 7.0, np.float32)
    small2 = np.full(10, 7.0, np.float32)
    rc = L.hifa4_calibration_load(bytes(p), ctypes.byref(hk), ctypes.byref(dd), ctypes.byref(al),
                                  small.ctypes.data_as(ctypes.c_void_p), small2.ctypes.data_as(ctypes.c_void_p), 10)
    assert rc == hifa4.ERR_INVALID_ARG and (hk.value, dd.value) == (2, 64)
    assert np.all(small == 7.0) and np.all(small2 == 7.0)
