"""Packed-weight files (mpw_file_*): host only.

* Round trip: matrices of several shapes, bit widths and both layouts come
  back byte for byte, with shape, width and layout.
* The bytes on disk follow the format the header documents, checked by an
  independent reader written here with struct and zlib's CRC-32.
* A matrix quantized and packed by the oracle unpacks to the same codes after
  the trip through a file.
* Corruption is reported: a flipped data byte or scale (checksum), a
  truncated file, a wrong magic or version, an index entry pointing past the
  end; a missing file is an I/O error; bad arguments are argument errors.
"""
import ctypes
import struct
import zlib

import numpy as np
import pytest
import torch

import mixed_precision_weight_row_b200 as mpw
import oracle


def _random_matrices(rng):
    mats = []
    for N, K, b, lay in [(3, 100, 5, "canonical"), (64, 512, 6, "paired"), (17, 96, 12, "paired"),
                         (1, 1, 4, "canonical"), (40, 4096, 15, "canonical"), (8, 64, 9, "paired")]:
        rb = mpw.packed_row_bytes(K, b)
        packed = torch.from_numpy(rng.integers(0, 256, size=(N, rb), dtype=np.uint8))
        scales = torch.from_numpy(rng.standard_normal(N).astype(np.float32))
        mats.append((packed, scales, b, K, lay))
    return mats


def test_round_trip(tmp_path):
    rng = np.random.default_rng(1)
    mats = _random_matrices(rng)
    path = str(tmp_path / "w.mpwpack")
    mpw.save_packed(path, mats)
    got = mpw.load_packed(path)
    assert len(got) == len(mats)
    for (packed, scales, b, K, lay), g in zip(mats, got):
        assert g["bits"] == b and g["K"] == K and g["N"] == packed.shape[0] and g["layout"] == lay
        assert torch.equal(g["packed"], packed)
        assert torch.equal(g["scales"].view(torch.int32), scales.view(torch.int32))


def _read_by_spec(path):
    """Independent reader of the documented layout."""
    data = open(path, "rb").read()
    magic, version, count, index_off, data_off = struct.unpack_from("<8sIIQQ", data, 0)
    assert magic == b"MPWPACK\0" and version == 1 and index_off == 32
    out = []
    for i in range(count):
        N, K, bits, layout, p_off, p_bytes, s_off, crc_p, crc_s, reserved = struct.unpack_from(
            "<QQIIQQQIIQ", data, 32 + 64 * i)
        assert reserved == 0
        assert p_off % 64 == 0 and s_off % 64 == 0 and p_off >= data_off and s_off >= p_off + p_bytes
        assert p_bytes == N * oracle.packed_row_bytes(K, bits)
        packed = data[p_off:p_off + p_bytes]
        scales = data[s_off:s_off + 4 * N]
        assert zlib.crc32(packed) == crc_p and zlib.crc32(scales) == crc_s
        out.append((N, K, bits, layout, packed, scales))
    assert len(data) % 64 == 0
    return out


def test_bytes_on_disk_follow_the_documented_format(tmp_path):
    rng = np.random.default_rng(2)
    mats = _random_matrices(rng)
    path = str(tmp_path / "w.mpwpack")
    mpw.save_packed(path, mats)
    recs = _read_by_spec(path)
    for (packed, scales, b, K, lay), (N, K2, b2, lay2, pbytes, sbytes) in zip(mats, recs):
        assert (N, K2, b2, lay2) == (packed.shape[0], K, b, mpw.LAYOUTS[lay])
        assert pbytes == packed.numpy().tobytes()
        assert sbytes == scales.numpy().astype("<f4").tobytes()


def test_oracle_codes_survive_a_file(tmp_path):
    rng = np.random.default_rng(3)
    W = rng.standard_normal((33, 320)).astype(np.float32) * np.float32(0.02)
    mats = []
    for b in (4, 7, 11):
        q, s = oracle.quantize(W, b)
        mats.append((torch.from_numpy(oracle.pack(q, b)), torch.from_numpy(s), b, 320, "canonical"))
        mats.append((torch.from_numpy(oracle.pack_paired(q, b)), torch.from_numpy(s), b, 320, "paired"))
    path = str(tmp_path / "codes.mpwpack")
    mpw.save_packed(path, mats)
    for g, b in zip(mpw.load_packed(path), (4, 4, 7, 7, 11, 11)):
        q, s = oracle.quantize(W, b)
        p = g["packed"].numpy()
        codes = oracle.unpack(p, 320, b) if g["layout"] == "canonical" else oracle.unpack_paired(p, 320, b)
        assert np.array_equal(codes, q)
        assert np.array_equal(g["scales"].numpy().view(np.uint32), s.view(np.uint32))


def _status_read(path, index=0):
    N, K, b, lay = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
    st = mpw.lib.mpw_file_info(path.encode(), index, ctypes.byref(N), ctypes.byref(K), ctypes.byref(b),
                               ctypes.byref(lay))
    if st != mpw.MPW_OK:
        return st
    packed = np.zeros(N.value * mpw.packed_row_bytes(K.value, b.value), dtype=np.uint8)
    scales = np.zeros(N.value, dtype=np.float32)
    return mpw.lib.mpw_file_read(path.encode(), index, packed.ctypes.data, scales.ctypes.data)


def test_corruption_is_reported(tmp_path):
    rng = np.random.default_rng(4)
    mats = _random_matrices(rng)[:2]
    path = str(tmp_path / "w.mpwpack")
    mpw.save_packed(path, mats)
    good = bytearray(open(path, "rb").read())
    _, _, _, _, p_off, p_bytes, s_off, _, _, _ = struct.unpack_from("<QQIIQQQIIQ", good, 32)
    assert _status_read(path) == mpw.MPW_OK

    def variant(name, blob):
        q = str(tmp_path / name)
        open(q, "wb").write(bytes(blob))
        return q

    flipped = bytearray(good)
    flipped[p_off + p_bytes // 2] ^= 0x10
    assert _status_read(variant("flip_packed", flipped)) == mpw.MPW_E_FORMAT
    flipped = bytearray(good)
    flipped[s_off + 1] ^= 0x01
    assert _status_read(variant("flip_scale", flipped)) == mpw.MPW_E_FORMAT
    assert _status_read(variant("truncated", good[: len(good) - 200])) == mpw.MPW_E_FORMAT
    assert _status_read(variant("header_only", good[:20])) == mpw.MPW_E_FORMAT
    bad = bytearray(good)
    bad[0:8] = b"NOTAPACK"
    assert _status_read(variant("magic", bad)) == mpw.MPW_E_FORMAT
    bad = bytearray(good)
    struct.pack_into("<I", bad, 8, 2)
    assert _status_read(variant("version", bad)) == mpw.MPW_E_FORMAT
    bad = bytearray(good)
    struct.pack_into("<Q", bad, 32 + 24, len(good) + 64)
    assert _status_read(variant("offset", bad)) == mpw.MPW_E_FORMAT
    assert _status_read(str(tmp_path / "missing.mpwpack")) == mpw.MPW_E_IO
    # an index past the count is an argument error, not a format error
    assert _status_read(path, index=5) == mpw.MPW_E_INVALID_ARG


def test_write_validation(tmp_path):
    L = mpw.lib
    buf = np.zeros(4096, dtype=np.uint8)
    sc = np.zeros(16, dtype=np.float32)
    path = str(tmp_path / "v.mpwpack").encode()

    def one(N, K, b, lay, packed=True, scales=True):
        arr = (mpw._FileMatrix * 1)()
        arr[0] = mpw._FileMatrix(N, K, b, lay, buf.ctypes.data if packed else None,
                                 sc.ctypes.data if scales else None)
        return L.mpw_file_write(path, arr, 1)

    assert one(4, 64, 3, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert one(4, 64, 16, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert one(0, 64, 5, 0) == mpw.MPW_E_INVALID_ARG
    assert one(4, 48, 5, 1) == mpw.MPW_E_INVALID_ARG        # paired needs K % 32 == 0
    assert one(4, 64, 5, 2) == mpw.MPW_E_INVALID_ARG
    assert one(4, 64, 5, 0, packed=False) == mpw.MPW_E_INVALID_ARG
    assert one(4, 64, 5, 0, scales=False) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_file_write(path, None, 1) == mpw.MPW_E_INVALID_ARG
    assert one(4, 64, 5, 0) == mpw.MPW_OK
    bad_dir = str(tmp_path / "no" / "such" / "dir" / "x").encode()
    arr = (mpw._FileMatrix * 1)()
    arr[0] = mpw._FileMatrix(4, 64, 5, 0, buf.ctypes.data, sc.ctypes.data)
    assert L.mpw_file_write(bad_dir, arr, 1) == mpw.MPW_E_IO
    with pytest.raises(ValueError):
        mpw.save_packed(str(tmp_path / "x"), [(torch.zeros((2, 7), dtype=torch.uint8), torch.zeros(2), 5, 64,
                                               "canonical")])
