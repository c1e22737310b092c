"""The product's lossless tile-ANS host encoder and blob validation (no GPU): byte-identical to the oracle's
blobs on every dtype, shape, tile size and bit-pattern family, independent of the thread count, and strict
about corrupt blobs."""
import numpy as np
import pytest
import torch

import decode_ep_b200 as ep
import oracle as orc

from test_oracle_tileans import DTYPES, SHAPES, bits_of

TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32, "fp8": torch.float8_e4m3fn,
         "int8": torch.int8}
VIEW = {"bf16": torch.int16, "fp16": torch.int16, "fp32": torch.int32, "fp8": torch.uint8, "int8": torch.uint8}


def tensor_of(kind: str, bits: np.ndarray) -> torch.Tensor:
    """The torch tensor whose raw bit patterns are `bits`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(torch.empty(0, dtype=VIEW[kind]).numpy().dtype).copy())
    return t.view(TORCH[kind]).reshape(bits.shape)


def several_coded_planes():
    """(kind, raw bits, K, coded planes mask) of tensors with two or more coded byte planes: values from a set of
    33 levels (every byte plane clusters), and FP32 copies of BF16 weights (zero low bytes and a clustered top
    byte coded around a raw one); one of them in ragged tiles of 7 elements a lane."""
    rng = np.random.default_rng(5)
    levels = torch.tensor(np.arange(-16, 17) / 8.0, dtype=torch.float32)
    idx = torch.from_numpy(rng.integers(0, 33, size=(3, 1000, 37)))
    cases = []
    for kind, mask in (("bf16", 3), ("fp16", 3), ("fp32", 15)):
        x = levels[idx].to(TORCH[kind])
        cases.append((kind, x.view(VIEW[kind]).numpy().view(np.uint32 if kind == "fp32" else np.uint16), 0, mask))
    y = (torch.from_numpy(rng.standard_normal((2000, 64))).float() * 0.02).to(torch.bfloat16).to(torch.float32)
    cases.append(("fp32", y.view(torch.int32).numpy().view(np.uint32), 0, 11))
    x = levels[torch.from_numpy(rng.integers(0, 33, size=(7, 3001)))].to(torch.bfloat16)
    cases.append(("bf16", x.view(torch.int16).numpy().view(np.uint16), 7, 3))
    return cases


def test_host_encoder_several_coded_planes():
    for kind, b, K, mask in several_coded_planes():
        c = ep.compress(tensor_of(kind, b), ep.TileANSConfig(elems_per_lane=K))
        assert ep.blob_info(c.blob)["coded_mask"] == mask, kind
        assert c.blob == orc.tans_compress(b, DTYPES[kind], K=K or 128), kind
        assert np.array_equal(orc.tans_decompress(c.blob), b), kind


@pytest.mark.parametrize("kind", list(DTYPES))
@pytest.mark.parametrize("shape", SHAPES)
def test_host_encoder_matches_oracle(kind, shape):
    b = bits_of(kind, shape, seed=len(shape) * 13 + DTYPES[kind])
    c = ep.compress(tensor_of(kind, b), ep.TileANSConfig())
    assert c.lossless and c.shape == tuple(shape) and c.dtype == TORCH[kind]
    assert c.blob == orc.tans_compress(b, DTYPES[kind])
    info = ep.blob_info(c.blob)
    want = orc.tans_info(c.blob)
    assert info["shape"] == want["shape"] and info["coded_mask"] == want["coded_mask"]


@pytest.mark.parametrize("K", [1, 7, 1024])
def test_host_encoder_tile_sizes_and_threads(K):
    b = bits_of("fp32", (3, 5000), seed=K)
    blobs = {ep.compress(tensor_of("fp32", b), ep.TileANSConfig(elems_per_lane=K, threads=t)).blob for t in (1, 3, 0)}
    assert blobs == {orc.tans_compress(b, 3, K=K)}


def test_host_encoder_special_patterns_and_distributions():
    rng = np.random.default_rng(9)
    cases = [("bf16", np.array([0x7FC1, 0xFF81, 0x7F80, 0x0000, 0x8000, 0x0001] * 700, np.uint16)),
             ("fp32", rng.integers(0, 2**32, size=9000, dtype=np.uint64).astype(np.uint32)),
             ("int8", np.full((70, 70), 3, np.uint8)),
             ("fp16", bits_of("fp16", (100, 100), seed=2, scale=1e4)),
             ("bf16", bits_of("bf16", (64, 1000), seed=7, scale=1e-30))]
    for kind, b in cases:
        c = ep.compress(tensor_of(kind, b), ep.TileANSConfig())
        assert c.blob == orc.tans_compress(b, DTYPES[kind]), kind


def test_validation_rejects_corrupt_blobs():
    b = bits_of("bf16", (20000,), seed=4)
    blob = bytearray(ep.compress(tensor_of("bf16", b), ep.TileANSConfig()).blob)
    for pos in (5, 8, 48, 52, 100):  # version, numel, K, tiles, a table frequency (CRC)
        bad = bytearray(blob)
        bad[pos] ^= 0x11
        with pytest.raises(ep.EntroPackError):
            ep.blob_info(bytes(bad))
    with pytest.raises(ep.EntroPackError):
        ep.blob_info(bytes(blob[:-16]))
    with pytest.raises(ep.EntroPackError):
        ep.compress(torch.zeros(2, 3, dtype=torch.float64), ep.TileANSConfig())
    with pytest.raises(ep.EntroPackError):
        ep.compress(torch.zeros(2, 3, dtype=torch.bfloat16), ep.TileANSConfig(elems_per_lane=2000))


def test_ratio_on_bf16_weights():
    """Gaussian BF16 weights: the sign-and-exponent byte is coded, the mantissa byte raw: about 11 bits a
    value, the figure DFloat11 (prior art on the pages) reports for BF16 models."""
    b = bits_of("bf16", (1000, 1000), seed=1)
    c = ep.compress(tensor_of("bf16", b), ep.TileANSConfig())
    assert ep.blob_info(c.blob)["coded_mask"] == 0b10
    assert 10.0 < c.actual_bpp < 12.0
