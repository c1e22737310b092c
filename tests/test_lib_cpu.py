"""CPU-only checks of the product library (no GPU calls).

Covered here:
- libentropack.so loads and exports every function that include/entropack.h declares;
- the host encoder (product) and the oracle encoder are independent implementations of the same
  format, and they produce byte-identical blobs in both format versions;
- the host validator accepts every good blob and rejects corrupted ones;
- the C ABI returns the documented status codes for bad input (README, Config table: the target
  range; 2-D only).
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ep():
    import decode_ep_b200 as m
    m.lib()
    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "entropack.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(ep):
    names = declared_functions()
    assert len(names) >= 10
    L = ctypes.CDLL(ep.lib()._name)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/entropack.h but not exported"


def test_library_is_sm100a_build(ep):
    import decode_ep_b200.build as b
    assert "arch=compute_100a,code=sm_100a" in " ".join(b.ARCH)
    assert os.path.dirname(ep.lib()._name) == os.path.join(ROOT, "decode_ep_b200")


CASES = [
    ("quickstart", lambda: synth.quickstart_256(), 3.5, 16),
    ("outliers", lambda: synth.lognormal_rows_with_outliers(n=256, seed=11, outlier_frac=2e-3, outlier_mult=40.0), 4.0, 16),
    ("fp16_raw_bits", lambda: synth.gaussian(128, 128, seed=8, container="fp16"), 9.0, 16),
    ("ragged_1_group_tile", lambda: synth.gaussian(129, 8, seed=3, container="bf16"), 3.0, 2),
    ("fp8", lambda: synth.fp8_codes(64, 512, seed=3), 5.0, 16),
    ("int8", lambda: synth.int8_codes(64, 512, seed=4), 3.0, 16),
    ("fp32_11bpp", lambda: synth.gaussian(96, 64, seed=5, container="fp32"), 11.0, 16),
    ("all_zero", lambda: torch.zeros(64, 64, dtype=torch.bfloat16), 2.0, 16),
    ("below_floor", lambda: synth.gaussian(64, 64, seed=3, container="bf16"), 0.001, 16),
    ("dit_like", lambda: synth.dit_layer(3, shape=(512, 256)), 4.0, 16),
    ("G1024", lambda: synth.gaussian(200, 96, seed=9, container="bf16"), 2.5, 1024),
]


PBITS = {1: 12, 2: 8}  # format version -> frequency precision


@pytest.mark.parametrize("version", [2, 1])
@pytest.mark.parametrize("name,maker,target,G", CASES, ids=[c[0] for c in CASES])
def test_host_encoder_matches_oracle_bytes(ep, orc, name, maker, target, G, version):
    w = maker()
    ob, obpp = orc.compress(synth.container_bits(w), synth.dtype_code(w), target, G, prob_bits=PBITS[version])
    c = ep.compress(w, ep.EntroPackLossyConfig(target, rounds_per_tile=G, format_version=version))
    assert c.blob == ob
    assert orc.blob_info(c.blob)["version"] == version
    assert c.actual_bpp == pytest.approx(obpp)
    info = ep.blob_info(c.blob)
    assert (info["rows"], info["cols"]) == tuple(w.shape)
    assert orc.blob_info(c.blob)["num_tiles"] >= 1


def test_host_encoder_thread_count_does_not_change_the_blob(ep):
    w = synth.dit_layer(5, shape=(300, 512))
    blobs = {ep.compress(w, ep.EntroPackLossyConfig(3.7, threads=t)).blob for t in (1, 3, 8)}
    assert len(blobs) == 1


def test_strided_input(ep):
    base = synth.gaussian(64, 96, seed=12, container="bf16")
    view = base[:, 16:80]
    assert view.stride(0) == 96
    a = ep.compress(view, 3.0).blob
    b = ep.compress(view.contiguous(), 3.0).blob
    assert a == b
    # Views whose rows are not dense (row stride below cols) are copied before encoding.
    row = synth.gaussian(1, 64, seed=13, container="bf16")
    expanded = row.expand(8, 64)
    assert expanded.stride(0) == 0
    assert ep.compress(expanded, 4.0).blob == ep.compress(expanded.contiguous(), 4.0).blob
    transposed = synth.gaussian(64, 32, seed=14, container="bf16").t()
    assert ep.compress(transposed, 4.0).blob == ep.compress(transposed.contiguous(), 4.0).blob


def test_status_codes(ep):
    w = synth.gaussian(16, 16, seed=1, container="bf16")
    for bad in (0.0009, 11.0001, float("nan"), float("inf")):
        with pytest.raises(ep.EntroPackError) as e:
            ep.compress(w, bad)
        assert e.value.status == -4
    with pytest.raises(ep.EntroPackError) as e:
        ep.compress(torch.zeros(4, 12, dtype=torch.bfloat16), 3.0)
    assert e.value.status == -3
    with pytest.raises(ep.EntroPackError) as e:
        ep.compress(torch.zeros(4, 4, 8, dtype=torch.bfloat16), 3.0)
    assert e.value.status == -3
    x = torch.zeros(8, 16)
    x[3, 3] = float("inf")
    with pytest.raises(ep.EntroPackError) as e:
        ep.compress(x, 3.0)
    assert e.value.status == -5
    L = ep.lib()
    assert L.ep_status_string(-6) == b"corrupt blob"


def test_validator_rejects_corruption(ep):
    c = ep.compress(synth.quickstart_256(), 3.5)
    ep.blob_info(c.blob)
    bad = bytearray(c.blob); bad[100] ^= 4          # scale byte: CRC
    with pytest.raises(ep.EntroPackError) as e:
        ep.blob_info(bytes(bad))
    assert e.value.status == -6
    with pytest.raises(ep.EntroPackError):
        ep.blob_info(c.blob[:-16])
    with pytest.raises(ep.EntroPackError):
        ep.blob_info(b"EPK1" + b"\0" * 60)


def test_decode_rejects_bad_arguments_without_launching(ep):
    """Host-side checks of ep_decompress_into run before any CUDA call."""
    c = ep.compress(synth.quickstart_256(), 3.5)
    L = ep.lib()
    hdr = c.header
    fake_dev = 0x10000  # never dereferenced: every case fails on the host first
    assert L.ep_decompress_into(hdr, fake_dev, len(c.blob) - 16, fake_dev, 1 << 20, None) == -9  # blob size
    assert L.ep_decompress_into(hdr, fake_dev + 8, len(c.blob), fake_dev, 1 << 20, None) == -9  # alignment
    assert L.ep_decompress_into(hdr, fake_dev, len(c.blob), fake_dev, 1000, None) == -9         # dst too small
    assert L.ep_decompress_into(b"EPK2" + hdr[4:], fake_dev, len(c.blob), fake_dev, 1 << 20, None) == -6
    assert L.ep_decompress_into(None, fake_dev, len(c.blob), fake_dev, 1 << 20, None) == -1


def test_decompress_many_checks_every_entry_before_launching(ep):
    """ep_decompress_many checks every header, size, pointer and alignment before its first CUDA call, whichever
    path the list takes (one sequence kernel, or one decode per blob for version-1 or mixed-dtype lists): a bad
    last entry is refused with nothing launched."""
    import ctypes as c
    L = ep.lib()
    w = synth.gaussian(64, 128, seed=21, container="bf16")
    v2 = ep.compress(w, 3.0)
    v1 = ep.compress(w, ep.EntroPackLossyConfig(3.0, format_version=1))
    f16 = ep.compress(synth.gaussian(64, 128, seed=22, container="fp16"), 3.0)
    comps = [v2, v1, f16]
    fake = 0x100000  # aligned and never dereferenced: every case fails on the host first

    def call(hdrs=None, blobs=None, sizes=None, dsts=None, dst_sizes=None, count=3):
        n = len(comps)
        H = (c.c_char_p * n)(*(hdrs or [x.header for x in comps]))
        B = (c.c_void_p * n)(*(blobs or [fake] * n))
        S = (c.c_size_t * n)(*(sizes or [len(x.blob) for x in comps]))
        D = (c.c_void_p * n)(*(dsts or [fake + 0x100000 * (k + 1) for k in range(n)]))
        Z = (c.c_size_t * n)(*(dst_sizes or [2 * 64 * 128] * n))
        return L.ep_decompress_many(count, H, B, S, D, Z, None)

    assert L.ep_decompress_many(-1, None, None, None, None, None, None) == -1
    assert L.ep_decompress_many(2, None, None, None, None, None, None) == -1
    assert L.ep_decompress_many(0, None, None, None, None, None, None) == 0
    good_dsts = [fake + 0x100000 * (k + 1) for k in range(3)]
    assert call(dsts=good_dsts[:2] + [good_dsts[2] + 8]) == -9            # last dst misaligned
    assert call(dst_sizes=[2 * 64 * 128, 2 * 64 * 128, 1000]) == -9        # last dst too small
    assert call(dsts=good_dsts[:2] + [None]) == -1                         # last dst NULL
    assert call(blobs=[fake, fake, fake + 4]) == -9                        # last blob misaligned
    assert call(sizes=[len(v2.blob), len(v1.blob) - 16, len(f16.blob)]) == -9  # a blob size mismatch
    assert call(hdrs=[v2.header, v1.header, b"EPKX" + f16.header[4:]]) == -6   # last header malformed
    assert L.ep_last_error().decode().startswith("ep_decompress_many")


def _fuzz_case(seed):
    """A seeded random tensor, target and tile size: shapes from one row to a few hundred, every container."""
    import random
    rnd = random.Random(seed)
    M, N = rnd.randint(1, 160), 8 * rnd.randint(1, 48)
    kind = rnd.choice(["bf16", "fp16", "fp32", "fp8", "int8", "outliers"])
    if kind == "fp8":
        w = synth.fp8_codes(M, N, seed=seed)
    elif kind == "int8":
        w = synth.int8_codes(M, N, seed=seed)
    elif kind == "outliers":
        w = synth.gaussian(M, N, seed=seed, container="fp32")
        w.view(-1)[:: max(1, (M * N) // 7)] *= 300.0  # a few escapes
        w = w.to(torch.bfloat16)
    else:
        w = synth.gaussian(M, N, seed=seed, std=rnd.choice([0.02, 1.0, 300.0]), container=kind)
    return w, round(rnd.uniform(0.3, 11.0), 3), rnd.choice([0, 1, 2, 5, 16, 40])


@pytest.mark.parametrize("version", [2, 1])
@pytest.mark.parametrize("seed", range(12))
def test_host_encoder_matches_oracle_bytes_fuzz(ep, orc, seed, version):
    w, target, G = _fuzz_case(1000 + seed)
    ob, _ = orc.compress(synth.container_bits(w), synth.dtype_code(w), target, G if G else 16,
                         prob_bits=PBITS[version])
    c = ep.compress(w, ep.EntroPackLossyConfig(target, rounds_per_tile=G if G else 16, format_version=version))
    assert c.blob == ob
