"""Compact PTQ state record (hif4_ptq_state_*): the serialized codes, metadata,
protected-column indices and BF16 protected weights of one linear layer
[TA summary, "Method overview": compact deltas restore the quantized
behaviour instead of full BF16 weights].

The record is checked against its documented version-1 layout by an
independent parser written here (struct + numpy), its checksum against
zlib's CRC-32, and every kind of damage (any flipped byte, truncation, a
wrong magic or version, unsorted indices) must be refused.  The codes and
metadata come from the CPU oracle, so these tests need no GPU; the last one
restores a GPU-quantized layer and checks the linear output bit for bit.
"""
import ctypes
import struct
import zlib

import numpy as np
import pytest

import oracle
from block_floating_point_hif4_b200 import workloads as wl


@pytest.fixture(scope="module")
def B():
    from block_floating_point_hif4_b200 import build
    build.build()
    from block_floating_point_hif4_b200 import binding
    binding.lib()
    return binding


def _a64(v):
    return (v + 63) // 64 * 64


def make_layer(N, K, n_masked, seed):
    rng = np.random.default_rng(seed)
    w = wl.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    idx = np.sort(rng.choice(K, n_masked, replace=False)).astype(np.int32)
    cm = np.zeros(K, np.uint8)
    cm[idx] = 1
    codes, meta, _ = oracle.quantize(w, cm)
    return codes, meta, idx, np.ascontiguousarray(w[:, idx])


def pack(B, codes, meta, idx, wm):
    import torch
    return B.ptq_state_pack(torch.from_numpy(codes), torch.from_numpy(meta.view(np.int32)),
                            torch.from_numpy(idx) if len(idx) else None,
                            torch.from_numpy(wm.view(np.int16)).view(torch.bfloat16) if len(idx) else None)


def parse_v1(rec: bytes):
    """Independent reader of the documented version-1 layout."""
    magic, ver, hdr, N, K, nm, flags, total = struct.unpack_from("<8sIIqqiIQ", rec, 0)
    assert magic == b"HIF4PTQS" and ver == 1 and hdr == 64 and flags == 0
    assert rec[48:64] == bytes(16)
    o_idx = 64
    o_codes = _a64(o_idx + 4 * nm)
    o_meta = _a64(o_codes + N * K // 2)
    o_wm = _a64(o_meta + 4 * N * (K // 64))
    o_crc = _a64(o_wm + 2 * N * nm)
    assert total == o_crc + 4 == len(rec)
    idx = np.frombuffer(rec, np.int32, nm, o_idx)
    codes = np.frombuffer(rec, np.uint8, N * K // 2, o_codes).reshape(N, K // 2)
    meta = np.frombuffer(rec, np.uint32, N * (K // 64), o_meta).reshape(N, K // 64)
    wm = np.frombuffer(rec, np.uint16, N * nm, o_wm).reshape(N, nm)
    crc = struct.unpack_from("<I", rec, o_crc)[0]
    return N, K, idx, codes, meta, wm, crc, o_crc


@pytest.mark.parametrize("N,K,nm", [(1, 64, 0), (37, 320, 3), (130, 1024, 10)])
def test_record_matches_documented_layout_and_round_trips(B, N, K, nm):
    import torch
    codes, meta, idx, wm = make_layer(N, K, nm, seed=N + K)
    rec = pack(B, codes, meta, idx, wm)
    assert len(rec) == B.lib().hif4_ptq_state_bytes(N, K, nm)
    n2, k2, i2, c2, m2, w2, crc, o_crc = parse_v1(rec)
    assert (n2, k2) == (N, K)
    assert np.array_equal(i2, idx) and np.array_equal(c2, codes) and np.array_equal(m2, meta)
    assert np.array_equal(w2, wm)
    assert crc == zlib.crc32(rec[:o_crc]) & 0xFFFFFFFF
    c3, m3, i3, w3 = B.ptq_state_unpack(rec)
    assert np.array_equal(c3.numpy(), codes) and np.array_equal(m3.numpy().view(np.uint32), meta)
    if nm:
        assert np.array_equal(i3.numpy(), idx)
        assert np.array_equal(w3.view(torch.int16).numpy().view(np.uint16), wm)
    else:
        assert i3 is None and w3 is None


def _info(B, rec):
    buf = ctypes.create_string_buffer(bytes(rec), len(rec))
    return B.lib().hif4_ptq_state_info(ctypes.cast(buf, ctypes.c_void_p), len(rec), None, None, None)


def _with_crc(rec: bytearray):
    o_crc = len(rec) - 4
    struct.pack_into("<I", rec, o_crc, zlib.crc32(bytes(rec[:o_crc])) & 0xFFFFFFFF)
    return rec


def test_damaged_records_are_refused(B):
    codes, meta, idx, wm = make_layer(20, 256, 4, seed=3)
    rec = pack(B, codes, meta, idx, wm)
    assert _info(B, rec) == 0
    rng = np.random.default_rng(4)
    # a flipped bit anywhere (header, every section, padding, checksum)
    for pos in list(range(0, 64, 3)) + list(rng.integers(64, len(rec), 200)) + [len(rec) - 1]:
        bad = bytearray(rec)
        bad[pos] ^= 1 << int(rng.integers(0, 8))
        assert _info(B, bad) == 9, pos
    # truncated anywhere; trailing bytes past the stated size are not part of the record
    assert _info(B, rec + b"\x00" * 7) == 0
    assert _info(B, rec[:-1]) == 9
    assert _info(B, rec[:64]) == 9
    assert _info(B, b"") == 9
    # a consistent checksum does not rescue a wrong magic, version or unsorted indices
    bad = bytearray(rec)
    bad[0:8] = b"HIF4PTQX"
    assert _info(B, _with_crc(bad)) == 9
    bad = bytearray(rec)
    struct.pack_into("<I", bad, 8, 2)
    assert _info(B, _with_crc(bad)) == 9
    bad = bytearray(rec)
    struct.pack_into("<ii", bad, 64, int(idx[1]), int(idx[0]))
    assert _info(B, _with_crc(bad)) == 9
    bad = bytearray(rec)
    struct.pack_into("<i", bad, 64, 256)                   # index out of range
    assert _info(B, _with_crc(bad)) == 9


def test_pack_argument_errors(B):
    L = B.lib()
    P = ctypes.c_void_p
    buf = ctypes.create_string_buffer(1 << 16)
    dst = ctypes.cast(buf, P)
    codes = (ctypes.c_uint8 * 4096)()
    meta = (ctypes.c_uint32 * 64)()
    idx = (ctypes.c_int32 * 2)(5, 3)
    wm = (ctypes.c_uint16 * 64)()
    assert L.hif4_ptq_state_pack(4, 100, codes, meta, None, 0, None, dst, 1 << 16) == 3      # K % 64
    assert L.hif4_ptq_state_pack(4, 128, codes, meta, idx, 2, wm, dst, 1 << 16) == 1          # unsorted
    assert L.hif4_ptq_state_pack(4, 128, codes, meta, None, 2, None, dst, 1 << 16) == 1       # missing idx
    assert L.hif4_ptq_state_pack(4, 128, codes, meta, None, 0, None, dst, 100) == 4           # too small
    assert L.hif4_ptq_state_pack(0, 128, codes, meta, None, 0, None, dst, 1 << 16) == 1
    assert L.hif4_ptq_state_bytes(4, 100, 0) == 0 and L.hif4_ptq_state_bytes(4, 128, 129) == 0


def test_wan22_record_sizes(B):
    """The records of the Wan2.2 FFN weights against their BF16 size."""
    L = B.lib()
    for N, K, nm in [(13824, 5120, 51), (5120, 13824, 138)]:
        size = L.hif4_ptq_state_bytes(N, K, nm)
        assert size == _a64(_a64(_a64(_a64(64 + 4 * nm) + N * K // 2) + 4 * N * K // 64) + 2 * N * nm) + 4
        assert size < 0.31 * (2 * N * K)                   # 4.5 bits per weight + protected columns


@pytest.mark.gpu
def test_restored_layer_gives_the_same_linear(B):
    import torch
    M, N, K = 300, 512, 1024
    rng = np.random.default_rng(9)
    x = torch.from_numpy(wl.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)).view(np.int16))
    x = x.view(torch.bfloat16).cuda()
    w_bits = wl.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.03).astype(np.float32))
    idx = np.sort(rng.choice(K, 10, replace=False)).astype(np.int32)
    cm = np.zeros(K, np.uint8)
    cm[idx] = 1
    w = torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16).cuda()
    codes, meta = B.quantize(w, torch.from_numpy(cm).cuda())
    i_dev = torch.from_numpy(idx).cuda()
    wm = w[:, i_dev.long()].contiguous()
    y0 = B.linear_w4a4(x, codes, meta, N, i_dev, wm)
    rec = B.ptq_state_pack(codes, meta, i_dev, wm)
    c2, m2, i2, w2 = B.ptq_state_unpack(rec, device="cuda")
    y1 = B.linear_w4a4(x, c2, m2, N, i2, w2)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert len(rec) < 0.31 * 2 * N * K
