"""GPU parity of the lossless tile-ANS decode (ep_tans_decompress_into, through the C ABI) with the CPU
oracle: every element's bit pattern identical, on every dtype, shape and tile size, on full-size tensors, and
the kernel's own checks of corrupt blobs (status bits, no fault)."""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import decode_ep_b200 as ep  # noqa: E402

from test_oracle_tileans import DTYPES, SHAPES, bits_of  # noqa: E402
from test_tans_cpu import VIEW, several_coded_planes, tensor_of  # noqa: E402


def raw_bits(t: torch.Tensor, kind: str) -> np.ndarray:
    return t.cpu().view(VIEW[kind]).numpy().view(bits_dtype(kind))


def bits_dtype(kind):
    return {"bf16": np.uint16, "fp16": np.uint16, "fp32": np.uint32, "fp8": np.uint8, "int8": np.uint8}[kind]


def status_clean():
    assert ep.device_status() == 0


def oracle_parallel(orc, blob: bytes, shape, dt):
    """The oracle's decode, its independent tiles spread over the host's cores."""
    info = orc.tans_info(blob)
    out = np.zeros(shape, dt)
    T = info["num_tiles"]
    step = max(1, T // (4 * (os.cpu_count() or 1)))
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(lambda a: orc.tans_decode_tiles(blob, a, min(T, a + step), out), range(0, T, step)))
    return out


@pytest.mark.parametrize("kind", list(DTYPES))
@pytest.mark.parametrize("shape", SHAPES)
def test_decode_matches_oracle(orc, kind, shape):
    b = bits_of(kind, shape, seed=len(shape) * 5 + DTYPES[kind])
    c = ep.compress(tensor_of(kind, b), ep.TileANSConfig())
    got = ep.decompress(c)
    status_clean()
    assert got.shape == tuple(shape) and got.dtype == c.dtype
    assert np.array_equal(raw_bits(got, kind), orc.tans_decompress(c.blob))


@pytest.mark.parametrize("K", [1, 7, 1024])
def test_decode_tile_sizes(orc, K):
    for kind in ("bf16", "fp32", "int8"):
        b = bits_of(kind, (7, 3001), seed=K)
        c = ep.compress(tensor_of(kind, b), ep.TileANSConfig(elems_per_lane=K))
        got = ep.decompress(c)
        status_clean()
        assert np.array_equal(raw_bits(got, kind), orc.tans_decompress(c.blob))


def test_decode_several_coded_planes(orc):
    """Tiles with two to four rANS-coded byte planes, each decoded from the lane's one state in plane order
    (coded masks 3, 15 and 11, a raw plane between coded ones included, and ragged tiles of 7 elements a
    lane): every element against the oracle and the input."""
    for kind, b, K, mask in several_coded_planes():
        c = ep.compress(tensor_of(kind, b), ep.TileANSConfig(elems_per_lane=K))
        assert ep.blob_info(c.blob)["coded_mask"] == mask
        got = ep.decompress(c)
        status_clean()
        assert np.array_equal(raw_bits(got, kind), orc.tans_decompress(c.blob))
        assert np.array_equal(raw_bits(got, kind), b)


def test_decode_special_patterns_and_all_raw(orc):
    rng = np.random.default_rng(3)
    cases = [("bf16", np.array([0x7FC1, 0xFF81, 0x7F80, 0x0000, 0x8000, 0x0001] * 5000, np.uint16)),
             ("fp32", rng.integers(0, 2**32, size=100_000, dtype=np.uint64).astype(np.uint32)),
             ("int8", np.full((300, 300), 3, np.uint8))]
    for kind, b in cases:
        c = ep.compress(tensor_of(kind, b), ep.TileANSConfig())
        got = ep.decompress(c)
        status_clean()
        assert np.array_equal(raw_bits(got, kind), b)


@pytest.mark.parametrize("kind,shape", [("bf16", (4, 4096, 4096)), ("fp32", (8192, 8192)), ("fp16", (64, 1024, 1024)),
                                        ("fp8", (8192, 28672)), ("int8", (8192, 28672))])
def test_full_size_every_element(orc, kind, shape):
    b = bits_of(kind, shape, seed=17)
    c = ep.compress(tensor_of(kind, b), ep.TileANSConfig())
    got = ep.decompress(c)
    status_clean()
    assert np.array_equal(raw_bits(got, kind), oracle_parallel(orc, c.blob, shape, bits_dtype(kind)))
    assert np.array_equal(raw_bits(got, kind), b)


def test_corrupt_blobs_set_status_bits(orc):
    """Host checks catch the header; the kernel catches the rest: a flipped word-stream byte fails the end-of-tile
    check, a zeroed table fails the table sum, a broken tile offset is refused; the context stays usable."""
    b = bits_of("bf16", (50_000,), seed=8)
    good = ep.compress(tensor_of("bf16", b), ep.TileANSConfig())
    out = torch.empty(good.shape, dtype=good.dtype, device="cuda")
    status_clean()
    off_tables = int.from_bytes(good.blob[56:60], "little")
    off_offsets = int.from_bytes(good.blob[60:64], "little")
    cases = []
    bad = bytearray(good.blob)
    bad[len(bad) - 64] ^= 0xA5  # the last tile's word stream
    cases.append((bytes(bad), 1))  # EP_DEV_CORRUPT_TILE
    bad = bytearray(good.blob)
    bad[off_tables + 4: off_tables + 12] = bytes(8)  # frequencies no longer sum to 4096
    cases.append((bytes(bad), 4 | 1))  # EP_DEV_BAD_TABLES (and the tiles then fail)
    bad = bytearray(good.blob)
    bad[off_offsets + 4: off_offsets + 8] = (0x7FFFFFF).to_bytes(4, "little")
    cases.append((bytes(bad), 2))  # EP_DEV_BAD_OFFSETS
    for blob, bits in cases:
        ct = ep.CompressedTensor(blob, good.shape, good.dtype, good.actual_bpp)
        ep.decompress_into(ct, out)
        st = ep.device_status()
        assert st & bits and st != 0
    ep.decompress_into(good, out)
    status_clean()
    assert np.array_equal(raw_bits(out, "bf16"), b)
    with pytest.raises(ep.EntroPackError):
        ep.decompress_into(ep.CompressedTensor(good.blob[:-16], good.shape, good.dtype, 0.0), out)
