"""Pins of the oracle's lossless tile-ANS (EPL1) against what fixes it from outside: exact round trips of
every bit pattern, the layout's byte arithmetic, the ideal code length under the blob's own tables, the
plane rule and the frequency normalisation restated in numpy, and the entropy of the coded byte plane."""
import math

import numpy as np
import pytest
import torch

import oracle as orc

DTYPES = {"bf16": 1, "fp16": 2, "fp32": 3, "fp8": 4, "int8": 5}
ELEM = {1: 2, 2: 2, 3: 4, 4: 1, 5: 1}


def bits_of(kind: str, shape, seed: int, scale: float = 0.02) -> np.ndarray:
    """Raw bit patterns of seeded data of the container kind."""
    g = torch.Generator().manual_seed(seed)
    n = int(np.prod(shape)) if len(shape) else 1
    x = torch.randn(n, generator=g) * scale
    if kind == "bf16":
        b = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    elif kind == "fp16":
        b = x.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    elif kind == "fp32":
        b = x.numpy().view(np.uint32)
    elif kind == "fp8":
        b = (x * (448 / 0.1)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    else:
        b = (x * (32 / scale)).round().clamp(-127, 127).to(torch.int8).view(torch.uint8).numpy()
    return b.reshape(shape).copy()


def pad16(n):
    return (n + 15) // 16 * 16


def pad4(n):
    return (n + 3) // 4 * 4


SHAPES = [(), (1,), (31,), (32,), (4096,), (4097,), (3, 70, 33), (2, 3, 4, 5, 6, 7, 1, 2), (0, 5), (5, 0)]


@pytest.mark.parametrize("kind", list(DTYPES))
@pytest.mark.parametrize("shape", SHAPES)
def test_tans_round_trip_every_dtype_and_shape(kind, shape):
    b = bits_of(kind, shape, seed=len(shape) * 7 + DTYPES[kind])
    blob = orc.tans_compress(b, DTYPES[kind])
    info = orc.tans_info(blob)
    assert info["shape"] == tuple(shape) and info["dtype"] == DTYPES[kind]
    assert np.array_equal(orc.tans_decompress(blob), b)


@pytest.mark.parametrize("K", [1, 7, 128, 1024])
def test_tans_round_trip_tile_sizes(K):
    b = bits_of("bf16", (5000,), seed=K)
    blob = orc.tans_compress(b, 1, K=K)
    info = orc.tans_info(blob)
    assert info["K"] == K and info["num_tiles"] == math.ceil(5000 / (32 * K))
    assert np.array_equal(orc.tans_decompress(blob), b)
    # tiles decode on their own
    out = np.zeros_like(b)
    for t in reversed(range(info["num_tiles"])):
        orc.tans_decode_tiles(blob, t, t + 1, out)
    assert np.array_equal(out, b)


def test_tans_special_bit_patterns():
    """NaN payloads, signed zeros, infinities and subnormals come back bit for bit."""
    for dt, pats in [(1, [0x7FC1, 0xFF81, 0x7F80, 0xFF80, 0x0000, 0x8000, 0x0001, 0x807F, 0x7F7F]),
                     (2, [0x7E01, 0xFC00, 0x7C00, 0x8000, 0x0001, 0x83FF, 0x7BFF]),
                     (3, [0x7FC00001, 0xFF800000, 0x00000001, 0x80000000, 0x7F7FFFFF, 0x807FFFFF])]:
        a = np.array(pats * 300, dtype=orc.TANS_NP[dt])
        blob = orc.tans_compress(a, dt)
        assert np.array_equal(orc.tans_decompress(blob), a)


def test_tans_uniform_bytes_stay_raw_with_exact_size():
    """Uniform random patterns: no plane pays to code, and the blob size is the layout's arithmetic."""
    rng = np.random.default_rng(5)
    for dt in (1, 3, 5):
        n, K = 12345, 16
        a = rng.integers(0, np.iinfo(orc.TANS_NP[dt]).max + 1, size=n, dtype=np.uint64).astype(orc.TANS_NP[dt])
        blob = orc.tans_compress(a, dt, K=K)
        info = orc.tans_info(blob)
        assert info["coded_mask"] == 0
        T = math.ceil(n / (32 * K))
        e = ELEM[dt]
        tiles = sum(pad16(e * pad4(min(32 * K, n - 32 * K * t))) for t in range(T))
        assert len(blob) == pad16(96 + 4 * (T + 1)) + tiles
        assert np.array_equal(orc.tans_decompress(blob), a)


def test_tans_constant_tensor():
    """One value: every plane takes the single-symbol table (4095 and 1) and costs almost nothing."""
    a = np.full((64, 1000), 0x3F80, np.uint16)
    blob = orc.tans_compress(a, 1)
    info = orc.tans_info(blob)
    assert info["coded_mask"] == 0b11
    T = info["num_tiles"]
    # each tile: 128 B of states plus at most a few words of log2(4096/4095) bits per symbol
    assert len(blob) <= pad16(96 + 2 * 8) + pad16(4 * (T + 1)) + T * 144
    assert np.array_equal(orc.tans_decompress(blob), a)


def parse_tables(blob: bytes):
    """The coded planes' frequency tables, read from the bytes (independent of the oracle's parser)."""
    e = ELEM[blob[6]]
    mask = blob[50]
    off = int.from_bytes(blob[56:60], "little")
    tabs = {}
    for j in range(e):
        if not (mask >> j) & 1:
            continue
        lo = int.from_bytes(blob[off:off + 2], "little")
        cnt = int.from_bytes(blob[off + 2:off + 4], "little")
        f = np.zeros(256, np.int64)
        f[lo:lo + cnt] = np.frombuffer(blob[off + 4:off + 4 + 2 * cnt], np.uint16)
        tabs[j] = f
        off += 4 + 2 * cnt
    return tabs


def planes(a: np.ndarray, e: int) -> np.ndarray:
    return np.ascontiguousarray(a).reshape(-1).view(np.uint8).reshape(-1, e)


def test_tans_coded_size_near_ideal():
    """The word streams take the ideal code length of the coded planes under the blob's own tables,
    within 1 % plus the tiles' fixed costs (the part of the stream the final states hold, padding)."""
    a = bits_of("bf16", (400_000,), seed=3)
    blob = orc.tans_compress(a, 1)
    info = orc.tans_info(blob)
    tabs = parse_tables(blob)
    assert set(tabs) == {1}
    pl = planes(a, 2)
    ideal_bits = 0.0
    for j, f in tabs.items():
        cnt = np.bincount(pl[:, j], minlength=256)
        assert np.all(f[cnt > 0] > 0) and f.sum() == 4096
        ideal_bits += float((cnt[cnt > 0] * np.log2(4096 / f[cnt > 0])).sum())
    T = info["num_tiles"]
    off_payload = int.from_bytes(blob[64:68], "little")
    payload = len(blob) - off_payload
    raw = sum(pad4(min(4096, a.size - 4096 * t)) for t in range(T))
    stream = payload - 128 * T - raw
    # A final state in [2^16, 2^32) holds up to 16 bits of the stream: at most 64 B a tile; padding adds < 16.
    assert ideal_bits / 8 - 64 * T <= stream <= 1.01 * ideal_bits / 8 + 16 * T


def normalize_np(counts: np.ndarray, M: int = 4096) -> np.ndarray:
    """The format document's normalisation (lossy section 7, item 3), restated."""
    f = np.zeros_like(counts)
    n, present = int(counts.sum()), np.flatnonzero(counts)
    if len(present) == 0:
        return f
    if len(present) == 1:
        s = int(present[0])
        f[s] = M - 1
        f[s + 1 if s + 1 < len(counts) else s - 1] = 1
        return f
    f[present] = np.maximum(1, counts[present] * M // n)
    d = M - int(f.sum())
    while d != 0:
        best = int(np.argmax(np.where(f > 0, f, -1)))
        if d > 0:
            f[best] += d
            d = 0
        else:
            take = min(-d, int(f[best]) - 1)
            f[best] -= take
            d += take
    return f


@pytest.mark.parametrize("kind,scale", [("bf16", 0.02), ("bf16", 1e3), ("fp16", 0.02), ("fp32", 0.02),
                                         ("fp8", 0.02), ("int8", 0.02), ("int8", 1e-4)])
def test_tans_plane_rule_matches_restatement(kind, scale):
    """Which planes are coded, and with which tables: the rule of the format document computed in numpy."""
    a = bits_of(kind, (50_000,), seed=11, scale=scale)
    dt = DTYPES[kind]
    blob = orc.tans_compress(a, dt)
    mask, tabs = orc.tans_info(blob)["coded_mask"], parse_tables(blob)
    pl = planes(a, ELEM[dt])
    want = 0
    for j in range(ELEM[dt]):
        cnt = np.bincount(pl[:, j], minlength=256).astype(np.int64)
        f = normalize_np(cnt)
        nz = np.flatnonzero(f)
        cost = 8.0 * (4 + 2 * (nz[-1] - nz[0] + 1)) + float((cnt[cnt > 0] * np.log2(4096 / f[cnt > 0])).sum())
        if cost <= 7.0 * len(pl):
            want |= 1 << j
            assert np.array_equal(tabs[j], f)
    assert mask == want


def test_tans_bf16_near_high_byte_entropy():
    """On Gaussian BF16 weights only the high byte (sign and seven exponent bits) is coded: the blob takes
    8 bits for the low byte plus about the high byte's entropy per element."""
    a = bits_of("bf16", (1_000_000,), seed=21)
    blob = orc.tans_compress(a, 1)
    hb = planes(a, 2)[:, 1]
    p = np.bincount(hb, minlength=256) / hb.size
    H = float(-(p[p > 0] * np.log2(p[p > 0])).sum())
    bits = 8 * len(blob) / a.size
    assert 8 + H <= bits <= 8 + H + 0.35
    assert bits < 12


def test_tans_corruption_is_detected():
    a = bits_of("bf16", (20_000,), seed=4)
    blob = bytearray(orc.tans_compress(a, 1))
    off_payload = int.from_bytes(blob[64:68], "little")
    bad = bytearray(blob)
    bad[len(bad) - 40] ^= 0x5A  # inside the last tile's word stream
    with pytest.raises(orc.OracleError):
        orc.tans_decompress(bytes(bad))
    bad = bytearray(blob)
    bad[100] ^= 1  # a table frequency: the CRC catches it
    with pytest.raises(orc.OracleError):
        orc.tans_info(bytes(bad))
    with pytest.raises(orc.OracleError):
        orc.tans_info(bytes(blob[: off_payload + 16]))
