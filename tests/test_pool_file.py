"""The packed pool as a file (Figure 1 caption: the experts are quantised
and packed ahead of time): host-only save / load through the C ABI, on the CPU. The file
format stated in include/exactmoe.h is checked independently here: the header
fields are parsed with `struct` and the checksum is recomputed with numpy."""
import os
import struct

import numpy as np
import pytest


@pytest.fixture(scope="module")
def N():
    from w4a16_mixture_experts_moe_b200 import build
    build.build()
    from w4a16_mixture_experts_moe_b200 import _native
    return _native


def _fnv1a_words(payload: bytes) -> int:
    h = 0xcbf29ce484222325
    for w in np.frombuffer(payload, dtype="<u8").tolist():
        h = ((h ^ w) * 0x100000001b3) & 0xFFFFFFFFFFFFFFFF
    return h


def _pool(layers, E, rec, seed=0):
    return np.random.default_rng(seed).integers(0, 256, size=layers * E * rec, dtype=np.uint8)


def test_round_trip_header_and_checksum(N, tmp_path):
    layers, E, H, I = 2, 3, 256, 256
    rec = N.moe_expert_record_layout(H, I)["bytes"]
    pool = _pool(layers, E, rec)
    path = str(tmp_path / "pool.bin")
    N.moe_pool_save(path, layers, E, H, I, rec, pool)
    raw = open(path, "rb").read()
    assert len(raw) == 64 + pool.size
    magic, ver, hdr, l_, e_, h_, i_, rb, pb, cs, zero = struct.unpack("<8sIIiiiiqqQQ", raw[:64])
    assert (magic, ver, hdr, l_, e_, h_, i_, rb, pb, zero) == (b"EXMOEPK1", 1, 64, layers, E, H, I, rec, pool.size, 0)
    assert raw[64:] == pool.tobytes()
    assert cs == _fnv1a_words(raw[64:])
    assert N.moe_pool_file_info(path) == {"layers": layers, "E": E, "H": H, "I": I, "record_bytes": rec}
    out = np.zeros_like(pool)
    info = N.moe_pool_load(path, out, out.size)
    assert info["record_bytes"] == rec and np.array_equal(out, pool)
    assert not os.path.exists(path + ".tmp")


def test_corrupt_truncated_and_mismatched_files_are_rejected(N, tmp_path):
    layers, E, H, I = 1, 2, 128, 256
    rec = N.moe_expert_record_layout(H, I)["bytes"]
    pool = _pool(layers, E, rec, seed=1)
    path = str(tmp_path / "pool.bin")
    N.moe_pool_save(path, layers, E, H, I, rec, pool)
    good = open(path, "rb").read()
    out = np.zeros_like(pool)

    def expect(data, status, text):
        bad = str(tmp_path / "bad.bin")
        open(bad, "wb").write(data)
        with pytest.raises(N.MoeError) as ei:
            N.moe_pool_load(bad, out, out.size)
        assert ei.value.status == status and text in str(ei.value), str(ei.value)

    flipped = bytearray(good)
    flipped[64 + 1234] ^= 0x10
    expect(bytes(flipped), N.MOE_ERR_INVALID_ARG, "checksum")
    expect(good[:-100], N.MOE_ERR_INVALID_ARG, "truncated")
    expect(good + b"\0" * 8, N.MOE_ERR_INVALID_ARG, "past its records")
    expect(b"NOTAPOOL" + good[8:], N.MOE_ERR_INVALID_ARG, "magic")
    expect(good[:8] + struct.pack("<I", 2) + good[12:], N.MOE_ERR_UNSUPPORTED, "version")
    expect(good[:10], N.MOE_ERR_INVALID_ARG, "shorter than a pool header")
    with pytest.raises(N.MoeError) as ei:
        N.moe_pool_load(path, out, out.size - 1)
    assert "buffer" in str(ei.value)
    with pytest.raises(N.MoeError) as ei:                       # record too small for the shape
        N.moe_pool_save(path, layers, E, H, I, rec - 256, pool)
    assert ei.value.status == N.MOE_ERR_SHAPE
