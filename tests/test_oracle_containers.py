"""Pins for the oracle's container conversions.

The containers come from the paper page abstract (BF16, FP16, FP8 and INT8) and the README feature list (FP32).

Each conversion is pinned against an independent library routine:
- BF16 and FP16: torch CPU casts, which are IEEE round-to-nearest-even;
- FP8 e4m3: the torch float8_e4m3fn cast of values pre-clamped to ±448 (OCP e4m3, saturating);
- INT8: numpy rint, which rounds half to even, then a clamp.
"""
import numpy as np
import pytest
import torch


def interesting_floats(n=200000, seed=0):
    rng = np.random.default_rng(seed)
    parts = [
        rng.normal(size=n).astype(np.float32) * np.float32(0.02),
        rng.normal(size=n).astype(np.float32) * np.float32(300.0),
        (rng.normal(size=n) * 1e-5).astype(np.float32),
        rng.uniform(-1e5, 1e5, size=n).astype(np.float32),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 448.0, 464.0, 480.0, -500.0, 1e-8,
                  2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -9, 2.0 ** -10, 0.5, 1.5, 2.5, -0.5,
                  127.5, 128.5, -128.5, -129.0, 3.0e38], dtype=np.float32),
    ]
    # exact ties of each container: values halfway between neighbours
    k = rng.integers(0, 1 << 16, size=n).astype(np.uint32)
    parts.append(((k << 16) | 0x8000).view(np.float32))          # bf16 ties
    parts.append(np.round(rng.normal(size=n) * 50).astype(np.float32) + np.float32(0.5))  # int8 ties
    y = np.concatenate(parts)
    return y[np.isfinite(y)]


def test_bf16_matches_torch(orc):
    y = interesting_floats()
    got = orc.to_container(y, 1)
    want = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_fp16_matches_torch(orc):
    y = interesting_floats()
    got = orc.to_container(y, 2)
    want = torch.from_numpy(y).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_fp8_e4m3_saturating_matches_torch(orc):
    y = interesting_floats()
    got = orc.to_container(y, 4)
    want = torch.from_numpy(np.clip(y, -448.0, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch keeps the sign of a value that rounds to zero; so does the oracle
    assert np.array_equal(got, want)
    assert not np.any((got & 0x7F) == 0x7F)  # never NaN


def test_int8_round_half_even_clamp(orc):
    y = interesting_floats()
    got = orc.to_container(y, 5)
    want = np.clip(np.rint(y.astype(np.float64)), -128, 127).astype(np.int8)
    assert np.array_equal(got, want)


def test_fp32_identity(orc):
    y = interesting_floats()
    assert np.array_equal(orc.to_container(y, 3), y)


@pytest.mark.parametrize("dt,tdt", [(1, torch.bfloat16), (2, torch.float16), (4, torch.float8_e4m3fn),
                                    (5, torch.int8)])
def test_from_container_exact(orc, dt, tdt):
    """Every finite bit pattern decodes to the value torch assigns it."""
    if dt in (1, 2):
        bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
        t = torch.from_numpy(bits.view(np.int16)).view(tdt)
    else:
        bits = np.arange(256, dtype=np.uint16).astype(np.uint8)
        t = torch.from_numpy(bits).view(tdt) if dt == 4 else torch.from_numpy(bits.view(np.int8))
    ref = t.float().numpy()
    keep = np.isfinite(ref)
    got = orc.from_container(bits[keep] if dt != 5 else bits.view(np.int8)[keep], dt)
    assert np.array_equal(got, ref[keep])
    if (~keep).any():
        with pytest.raises(orc.OracleError):
            orc.from_container(bits[~keep][:1], dt)
