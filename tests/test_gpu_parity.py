"""GPU parity: the sm_100a decode (called through the C ABI) against the CPU oracle, on the same blobs.

The decode has to be bit-exact on two things:
- the lattice coordinates (z = 2v, from ep_decode_coords_into);
- the container values (ep_decompress_into). The reconstruction is fl32(v · fl32(s_row/α)),
  then the container rounding. Both sides compute it in IEEE binary32, so the bar is identity
  rather than the 1-ulp tolerance a looser reading of the rescale would need.

The blobs come from the product host encoder. A separate CPU test shows that encoder is
byte-identical to the oracle encoder.

Sizes:
- Small fuzz and edge cases, plus full-size tensors of every workload: 256², 3072² with
  outliers, each DiT-like layer shape, the 4096² bitrate sweep, and the 8192x28672 FP8/INT8
  codes.
- Every tile of every single-tensor workload is compared, the 8192x28672 code matrices and all 24
  sweep points included: the oracle decodes the tiles (which are independent) on all host cores.
- The full 276-layer sequence compares the first, a middle and the last (ragged) tile of every layer.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import decode_ep_b200 as ep  # noqa: E402

NP_BITS = {torch.bfloat16: np.uint16, torch.float16: np.uint16, torch.float32: np.float32,
           torch.float8_e4m3fn: np.uint8, torch.int8: np.int8}


def gpu_bits(t: torch.Tensor) -> np.ndarray:
    t = t.cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def status_clean():
    assert ep.device_status() == 0


def check_full(orc, c: ep.CompressedTensor):
    want, zwant = orc.decompress(c.blob, with_coords=True)
    got = gpu_bits(ep.decompress(c))
    z = ep.decode_coords(c).cpu().numpy()
    status_clean()
    assert np.array_equal(z, zwant), "lattice coordinates differ"
    if got.dtype == np.float32:
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    else:
        assert np.array_equal(got, want)


def oracle_decode_parallel(orc, blob: bytes, shape, np_dtype, with_coords=True, tiles=None):
    """The oracle's decode of the listed tiles (default: all), spread over the host's cores. Tiles are
    independent and write disjoint outputs; the oracle releases the GIL inside its C calls."""
    import concurrent.futures as cf
    import os
    info = orc.blob_info(blob)
    T = info["num_tiles"]
    want = np.zeros(shape, np_dtype)
    zwant = np.zeros(shape, np.int32) if with_coords else None
    if tiles is None:
        step = max(1, T // (4 * (os.cpu_count() or 1)))
        runs = [(j, min(T, j + step)) for j in range(0, T, step)]
    else:
        runs = [(int(j), int(j) + 1) for j in tiles]
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(lambda r: orc.decode_tiles(blob, r[0], r[1], want, zwant), runs))
    return want, zwant


def check_every_tile(orc, c: ep.CompressedTensor):
    """check_full with the oracle's decode spread over the host's cores, for the full-size tensors."""
    want, zwant = oracle_decode_parallel(orc, c.blob, c.shape, NP_BITS[c.dtype])
    got = gpu_bits(ep.decompress(c))
    z = ep.decode_coords(c).cpu().numpy()
    status_clean()
    assert np.array_equal(z, zwant), "lattice coordinates differ"
    if got.dtype == np.float32:
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    else:
        assert np.array_equal(got, want)


# ------------------------------------------------------------------- small and edge cases

EDGE = [
    ("quickstart", lambda: synth.quickstart_256(), 3.5, 16),
    ("outliers_esc", lambda: synth.lognormal_rows_with_outliers(n=256, seed=11, outlier_frac=2e-3, outlier_mult=40.0), 4.0, 16),
    ("fp16_raw_bits", lambda: synth.gaussian(128, 128, seed=8, container="fp16"), 9.0, 16),
    ("ragged_1_group_tile", lambda: synth.gaussian(129, 8, seed=3, container="bf16"), 3.0, 2),
    ("one_row", lambda: synth.gaussian(1, 8, seed=4, container="bf16"), 5.0, 1),
    ("narrow_rows", lambda: synth.gaussian(3000, 8, seed=13, container="bf16"), 4.0, 16),
    ("fp8", lambda: synth.fp8_codes(64, 512, seed=3), 5.0, 16),
    ("int8", lambda: synth.int8_codes(64, 512, seed=4), 3.0, 16),
    ("fp32_11bpp", lambda: synth.gaussian(96, 64, seed=5, container="fp32"), 11.0, 16),
    ("all_zero", lambda: torch.zeros(64, 64, dtype=torch.bfloat16), 2.0, 16),
    ("below_floor", lambda: synth.gaussian(64, 64, seed=3, container="bf16"), 0.001, 16),
    ("G1024", lambda: synth.gaussian(200, 96, seed=9, container="bf16"), 2.5, 1024),
    ("G1", lambda: synth.gaussian(40, 64, seed=10, container="fp16"), 6.0, 1),
]


VERSIONS = [2, 1]  # format version 2 (8-bit tables, the default) and version 1 (12-bit tables)


@pytest.mark.parametrize("version", VERSIONS)
@pytest.mark.parametrize("name,maker,target,G", EDGE, ids=[e[0] for e in EDGE])
def test_parity_edge_cases(orc, name, maker, target, G, version):
    c = ep.compress(maker(), ep.EntroPackLossyConfig(target, rounds_per_tile=G, format_version=version))
    check_full(orc, c)


@pytest.mark.parametrize("version", VERSIONS)
def test_parity_r12_extremes(orc, version):
    g = torch.Generator().manual_seed(6)
    w = torch.randn(40, 8, generator=g)
    c = ep.compress(w, ep.EntroPackLossyConfig(11.0, rounds_per_tile=1, format_version=version))
    check_full(orc, c)
    # int16-range escapes at r = 0 come from the oracle encoder with a forced alpha
    w2 = torch.randn(64, 4096, generator=g) * 1e-3
    w2[:, 7] = 1.0
    w2[::2, 9] = -1.0
    blob, _ = orc.compress(w2.numpy(), 3, 3.0, 16, 450.0, prob_bits=12 if version == 1 else 8)
    check_full(orc, ep.CompressedTensor.from_blob(blob))


def tile_mix(blob: bytes):
    """(r, tiles that hold an escape and fit the one-layer kernel's 5 KB tile buffer, tiles that fit
    without one, tiles too large for it): r is header byte 7, T the u32 at 24, the tile offsets (u32, in
    16-byte units, bit 31 set when the tile holds an escape) start at the u32 offset at 36."""
    import struct
    r = blob[7]
    T, = struct.unpack_from("<I", blob, 24)
    off, = struct.unpack_from("<I", blob, 36)
    offs = np.frombuffer(blob, np.uint32, T + 1, off).astype(np.int64)
    esc = (offs[:T] >> 31).astype(bool)
    start = offs & 0x7FFFFFFF
    fit = (start[1:] - start[:T]) * 16 <= 5 * 1024
    return r, int((esc & fit).sum()), int((~esc & fit).sum()), int((~fit).sum())


RAW_ESC = [
    # (id, container or None for an oracle-encoded int16-escape blob, rows, cols, target bpp, G or forced alpha)
    ("bf16_6bpp", "bf16", 1024, 2048, 6.0, 0),
    ("fp32_8bpp", "fp32", 1024, 2048, 8.0, 0),
    ("fp16_11bpp", "fp16", 1024, 2048, 11.0, 12),
    ("bf16_6bpp_rows_of_255_groups", "bf16", 1024, 2040, 6.0, 0),
    ("int16_escapes_r4", None, 64, 4096, 6.0, 100.0),
    ("int16_escapes_r7", None, 64, 4096, 6.0, 1000.0),
    ("int16_escapes_r4_rows_of_511_groups", None, 64, 4088, 6.0, 100.0),
]


@pytest.mark.parametrize("kind,cont,M,N,target,arg", RAW_ESC, ids=[e[0] for e in RAW_ESC])
def test_parity_raw_bit_tiles_with_escapes(orc, kind, cont, M, N, target, arg):
    """Tiles with raw low bits (r >= 1) decoded by the one-layer kernel's raw-bit fast rounds, with and
    without escapes, the escape rounds building integer values (escape words far outside the entries' +-31:
    |z| up to 128001 at r = 7), in rows of whole rounds and in rows that are not (255 and 511 groups). The
    blobs are checked to hold the kinds of tile asked for, whole in the tile buffer; every value and lattice
    coordinate is compared with the oracle."""
    if cont is None:
        g = torch.Generator().manual_seed(6)
        w = torch.randn(M, N, generator=g) * 1e-3
        w[:, 7] = 1.0
        w[::2, 9] = -1.0
        w[5::7, 100] = 0.5
        blob, _ = orc.compress(w.numpy(), 3, target, 16, arg)
        c = ep.CompressedTensor.from_blob(blob)
        r, esc_fit, plain_fit, too_big = tile_mix(blob)
        assert r == (4 if arg == 100.0 else 7) and esc_fit >= 60 and too_big == 0
    else:
        w = synth.gaussian(M, N, 41, container=cont)
        c = ep.compress(w, ep.EntroPackLossyConfig(target, rounds_per_tile=int(arg)))
        r, esc_fit, plain_fit, too_big = tile_mix(c.blob)
        assert r >= 1 and esc_fit >= 100 and plain_fit >= 100 and too_big == 0
    check_full(orc, c)


@pytest.mark.parametrize("version", VERSIONS)
def test_parity_random_fuzz(orc, version):
    rng = np.random.default_rng(2024)
    for it in range(30):
        M = int(rng.integers(1, 300)); N = 8 * int(rng.integers(1, 80))
        cont = ["bf16", "fp16", "fp32"][it % 3]
        w = synth.gaussian(M, N, seed=1000 + it, container=cont, std=float(rng.uniform(0.001, 3)))
        target = float(rng.uniform(0.3, 11.0))
        G = int(rng.choice([1, 2, 3, 16, 40]))
        check_full(orc, ep.compress(w, ep.EntroPackLossyConfig(target, rounds_per_tile=G, format_version=version)))


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("version", VERSIONS)
def test_parity_quickstart_256(orc, version):
    c = ep.compress(synth.quickstart_256(), ep.EntroPackLossyConfig(3.5, format_version=version))
    assert abs(c.actual_bpp - 3.5) <= 0.05
    out = ep.decompress(c)
    assert out.shape == (256, 256) and out.dtype == torch.bfloat16
    check_full(orc, c)


@pytest.mark.parametrize("version", VERSIONS)
def test_parity_3072_lognormal_outliers(orc, version):
    c = ep.compress(synth.lognormal_rows_with_outliers(), ep.EntroPackLossyConfig(4.0, format_version=version))
    assert c.actual_bpp <= 4.05
    check_every_tile(orc, c)


@pytest.mark.parametrize("version", VERSIONS)
@pytest.mark.parametrize("i", [0, 4, 6, 7, 272, 273, 274])
def test_parity_dit_layer_shapes(orc, i, version):
    """One layer of every distinct shape of the 276-layer DiT-like set, at 4 bpp."""
    w = synth.dit_layer(i)
    c = ep.compress(w, ep.EntroPackLossyConfig(4.0, format_version=version))
    assert c.actual_bpp <= 4.05
    check_every_tile(orc, c)


@pytest.mark.parametrize("version", VERSIONS)
def test_parity_bitrate_sweep_4096(orc, version):
    base = synth.gaussian(4096, 4096, seed=2, container="fp32")
    for cont in ("bf16", "fp16", "fp32"):
        w = base.to(synth.CONTAINERS[cont])
        prev = None
        for target in (0.5, 1.0, 2.3, 3.0, 5.0, 6.0, 8.0, 11.0):
            c = ep.compress(w, ep.EntroPackLossyConfig(target, format_version=version))
            assert abs(c.actual_bpp - target) <= 0.05
            check_every_tile(orc, c)
            y = ep.decompress(c).float()
            err = float((y - w.cuda().float()).norm() / w.cuda().float().norm())
            if prev is not None:
                assert err <= prev + 1e-7
            prev = err


@pytest.mark.parametrize("version", VERSIONS)
@pytest.mark.parametrize("kind", ["fp8", "int8"])
def test_parity_llm_prefill_containers(orc, kind, version):
    if kind == "fp8":
        w, target = synth.fp8_codes(), 5.0
    else:
        w, target = synth.int8_codes(), 3.0
    c = ep.compress(w, ep.EntroPackLossyConfig(target, format_version=version))
    assert abs(c.actual_bpp - target) <= 0.05
    check_every_tile(orc, c)


# -------------------------------------------------------------------- faults, made on the host

@pytest.mark.parametrize("version", VERSIONS)
def test_corrupt_payload_sets_status_not_fault(orc, version):
    c = ep.compress(synth.gaussian(512, 512, seed=3, container="bf16"), ep.EntroPackLossyConfig(4.0, format_version=version))
    off_payload = int.from_bytes(c.blob[40:44], "little")
    rng = np.random.default_rng(1)
    hits = 0
    for _ in range(12):
        bad = bytearray(c.blob)
        for _ in range(4):
            pos = int(rng.integers(off_payload + 128, len(bad)))
            bad[pos] ^= 0xFF
        cc = ep.CompressedTensor(bytes(bad), c.shape, c.dtype, c.actual_bpp)
        ep.decompress(cc)
        st = ep.device_status()
        hits += bool(st & 1)
    assert hits >= 11
    # the GPU keeps working after corrupt input
    check_full(orc, c)


@pytest.mark.parametrize("version", VERSIONS)
def test_corrupt_offsets_and_tables_flags(orc, version):
    c = ep.compress(synth.gaussian(512, 512, seed=4, container="bf16"), ep.EntroPackLossyConfig(4.0, format_version=version))
    hdr = c.blob[:64]
    off_tables = int.from_bytes(hdr[32:36], "little")
    off_offsets = int.from_bytes(hdr[36:40], "little")
    bad = bytearray(c.blob)
    bad[off_offsets + 4 * 5: off_offsets + 4 * 5 + 4] = (0x7FFFFFF0).to_bytes(4, "little")
    ep.decompress(ep.CompressedTensor(bytes(bad), c.shape, c.dtype, 0))
    assert ep.device_status() & 2
    bad = bytearray(c.blob)
    bad[off_tables + 17 + 3] = 200     # cnt beyond the alphabet
    bad[off_tables + 40] ^= 0x5A       # and a damaged frequency
    ep.decompress(ep.CompressedTensor(bytes(bad), c.shape, c.dtype, 0))
    assert ep.device_status() != 0
    check_full(orc, c)


def test_host_side_errors():
    c = ep.compress(synth.quickstart_256(), 3.5)
    out = torch.empty(255, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ep.EntroPackError) as e:
        ep.decompress_into(c, out)
    assert e.value.status == -9
    with pytest.raises(ep.EntroPackError):
        ep.decompress_into(c, torch.empty(256, 256, dtype=torch.float16, device="cuda"))


def test_streams_and_allocating_entry(orc):
    c = ep.compress(synth.dit_layer(9, shape=(512, 1024)), 4.0)
    s = torch.cuda.Stream()
    out = torch.empty(c.shape, dtype=c.dtype, device="cuda")
    with torch.cuda.stream(s):
        ep.decompress_into(c, out, stream=s)
    s.synchronize()
    ref = ep.decompress(c)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # ep_decompress allocates the output itself (cudaMallocAsync on the stream)
    from cuda.bindings import runtime as rt
    L = ep.lib()
    ptr = ctypes.c_void_p()
    dblob = c.device_blob()
    st = L.ep_decompress(c.header, dblob.data_ptr(), len(c.blob), ctypes.byref(ptr), None)
    assert st == 0 and ptr.value
    host = np.empty(c.shape, np.uint16)
    err, = rt.cudaMemcpy(host.ctypes.data, ptr.value, host.nbytes, rt.cudaMemcpyKind.cudaMemcpyDeviceToHost)
    assert err == rt.cudaError_t.cudaSuccess
    assert rt.cudaFree(ptr.value)[0] == rt.cudaError_t.cudaSuccess
    assert np.array_equal(host, gpu_bits(ref))


def test_decompress_many_matches_single_decodes(orc):
    """The layer-sequence entry in its launch-per-blob form (the list mixes format versions and dtypes)
    gives the same bytes as one-by-one decodes. The last output is one buffer shared by several layers,
    written in list order."""
    comps = [ep.compress(synth.dit_layer(i, shape=shp), 4.0)
             for i, shp in enumerate([(384, 256), (1024, 512), (64, 3840), (3840, 64), (1536, 256)])]
    comps.append(ep.compress(synth.fp8_codes(256, 512, seed=5), 5.0))
    comps.append(ep.compress(synth.gaussian(300, 200, seed=6, container="fp32"), 7.0))
    # version-1 blobs in the same sequence: their tables are prepared once, the others' built per CTA
    comps.append(ep.compress(synth.dit_layer(12, shape=(512, 512)), ep.EntroPackLossyConfig(4.0, format_version=1)))
    comps.append(ep.compress(synth.gaussian(96, 512, seed=7, container="bf16"), ep.EntroPackLossyConfig(6.0, format_version=1)))
    outs = [torch.empty(c.shape, dtype=c.dtype, device="cuda") for c in comps]
    batch = ep.LayerBatch(list(zip(comps, outs)))
    for _ in range(3):
        batch.run()
    status_clean()
    for c, o in zip(comps, outs):
        want = orc.decompress(c.blob)
        got = gpu_bits(o)
        if got.dtype == np.float32:
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
        else:
            assert np.array_equal(got, want)
    # one reused buffer: after the sequence it holds the last layer that wrote it
    shared = torch.empty(1024 * 512, dtype=torch.bfloat16, device="cuda")
    bf = [c for c in comps if c.dtype == torch.bfloat16]
    views = [shared[: c.shape[0] * c.shape[1]].view(c.shape) for c in bf]
    ep.decompress_many(list(zip(bf, views)))
    torch.cuda.synchronize()
    status_clean()
    last = bf[-1]
    assert np.array_equal(gpu_bits(views[-1]), orc.decompress(last.blob))


def test_planned_mixed_bitrate_sequence(orc):
    """Layers given per-layer targets by ep_plan_bitrates (a spread of rates, r > 0 on the top ones),
    encoded by the CUDA encoder, decoded as one sequence: every output equals the oracle's decode of
    the same blob, and the set's storage lands on the planned mean."""
    import math
    import random
    shapes = [(512, 256), (256, 1024), (64, 3840), (1024, 512), (384, 384), (3840, 64)]
    rnd = random.Random(3)
    sens = [math.exp(rnd.gauss(0.0, 2.0)) for _ in shapes]
    ws = [synth.dit_layer(40 + i, shape=s).cuda() for i, s in enumerate(shapes)]
    weights = [s * float(w.float().square().mean()) for s, w in zip(sens, ws)]
    mean = 3.0
    targets = ep.plan_bitrates(shapes, weights, mean)
    assert max(targets) - min(targets) > 2.0
    comps = [ep.compress(w, ep.EntroPackLossyConfig(t, encoder="cuda")) for w, t in zip(ws, targets)]
    outs = [torch.empty(c.shape, dtype=c.dtype, device="cuda") for c in comps]
    ep.LayerBatch(list(zip(comps, outs))).run()
    torch.cuda.synchronize()
    status_clean()
    for c, o in zip(comps, outs):
        assert np.array_equal(gpu_bits(o), orc.decompress(c.blob))
    n = sum(r * k for r, k in shapes)
    assert 8 * sum(len(c.blob) for c in comps) / n <= mean + 0.05


def test_table_copy_wait_runs_out_into_status(orc, monkeypatch):
    """The bounded wait for a sequence's table copies: with the copies left unissued (test hook), every
    CTA gives up, sets EP_DEV_TABLE_COPY and decodes nothing; the context stays usable."""
    # The prepared-table copies serve version-1 blobs (version-2 tables are built in each CTA).
    comps = [ep.compress(synth.gaussian(64, 256, seed=s, container="bf16"), ep.EntroPackLossyConfig(4.0, format_version=1))
             for s in (21, 22)]
    outs = [torch.zeros(c.shape, dtype=c.dtype, device="cuda") for c in comps]
    status_clean()
    monkeypatch.setenv("EPK_TEST_TABLE_COPY_TIMEOUT", "1")
    ep.decompress_many(list(zip(comps, outs)))
    st = ep.device_status()
    monkeypatch.delenv("EPK_TEST_TABLE_COPY_TIMEOUT")
    assert st & 8
    assert all(int(o.view(torch.int16).abs().sum()) == 0 for o in outs)  # nothing was stored
    ep.decompress_many(list(zip(comps, outs)))
    status_clean()
    for c, o in zip(comps, outs):
        assert np.array_equal(gpu_bits(o), orc.decompress(c.blob))


def test_decompress_many_edge_counts(orc):
    """Sequences of 0 and 1 blobs, and one longer than an expand launch takes (512 blobs): the tables are
    then prepared by two expand launches. Small mixed shapes and containers, each checked against the
    oracle."""
    ep.decompress_many([])
    status_clean()
    one = ep.compress(synth.gaussian(40, 64, seed=31, container="fp16"), 5.0)
    out1 = torch.empty(one.shape, dtype=one.dtype, device="cuda")
    ep.decompress_many([(one, out1)])
    status_clean()
    assert np.array_equal(gpu_bits(out1), orc.decompress(one.blob))
    comps = []
    for i in range(530):
        M, N = 1 + (i * 7) % 23, 8 * (1 + (i * 5) % 9)
        kind = ("bf16", "fp16", "fp32")[i % 3]
        comps.append(ep.compress(synth.gaussian(M, N, seed=1000 + i, container=kind),
                                 ep.EntroPackLossyConfig(1.0 + (i % 9), format_version=1 + i % 2)))
    outs = [torch.empty(c.shape, dtype=c.dtype, device="cuda") for c in comps]
    ep.decompress_many(list(zip(comps, outs)))
    torch.cuda.synchronize()
    status_clean()
    for c, o in zip(comps, outs):
        want = orc.decompress(c.blob)
        got = gpu_bits(o)
        if got.dtype == np.float32:
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
        else:
            assert np.array_equal(got, want)


@pytest.mark.slow
def test_full_276_layer_sequence_every_tile(orc):
    """The benchmark's launch configuration at full size: all 276 DiT-like layers (6.17 G parameters at
    4 bpp, CUDA encoder) decoded by one ep_decompress_many (the sequence kernel: one launch for all the
    layers), each layer into its own buffer. Every element of every layer is compared with the oracle's
    decode of the same blob, one layer at a time, the oracle's tiles spread over the host's cores."""
    import concurrent.futures as cf
    shapes = synth.dit_layer_shapes()
    with cf.ThreadPoolExecutor(max_workers=8) as ex:
        futs = [ex.submit(synth.dit_layer, i, (M, N)) for i, (_, M, N) in enumerate(shapes)]
        comps = []
        for f in futs:
            w = f.result().cuda()
            comps.append(ep.compress(w, ep.EntroPackLossyConfig(4.0, encoder="cuda")))
            del w
    outs = [torch.empty(c.shape, dtype=c.dtype, device="cuda") for c in comps]
    ep.decompress_many(list(zip(comps, outs)))
    torch.cuda.synchronize()
    status_clean()
    n = sum(M * N for _, M, N in shapes)
    assert 8 * sum(len(c.blob) for c in comps) / n <= 4.05
    for i, (c, o) in enumerate(zip(comps, outs)):
        want, _ = oracle_decode_parallel(orc, c.blob, c.shape, np.uint16, with_coords=False)
        assert np.array_equal(gpu_bits(o), want), f"layer {i}"


def test_version2_sequence_into_one_buffer_keeps_write_order(orc):
    """The sequence kernel orders its layers tile by tile: each tile waits only for the tiles of earlier layers
    that last wrote its bytes. Layers of mixed sizes decoded into one shared buffer (a small one between two large ones, so
    that a later layer overwrites a region the layer before it left alone) must leave, at every byte, the value
    of the last layer that wrote it. The expected buffer is assembled on the host from the oracle's decodes."""
    shapes = [(1024, 768), (96, 256), (768, 512), (64, 3840), (1536, 256), (256, 256), (1024, 640)]
    comps = [ep.compress(synth.dit_layer(60 + i, shape=s), ep.EntroPackLossyConfig(3.0 + 0.5 * (i % 3)))
             for i, s in enumerate(shapes)]
    assert all(int.from_bytes(c.blob[4:6], "little") == 2 for c in comps)
    total = max(M * N for M, N in shapes)
    shared = torch.zeros(total, dtype=torch.bfloat16, device="cuda")
    views = [shared[: M * N].view(M, N) for M, N in shapes]
    want = np.zeros(total, np.uint16)
    for c in comps:
        d = orc.decompress(c.blob).reshape(-1)
        want[: d.size] = d
    for _ in range(3):
        shared.zero_()
        ep.decompress_many(list(zip(comps, views)))
        torch.cuda.synchronize()
        status_clean()
        assert np.array_equal(gpu_bits(shared), want)


def _bits_any(t):
    b = gpu_bits(t)
    return b.view(np.uint32) if b.dtype == np.float32 else b


def _want_any(orc, c):
    w = orc.decompress(c.blob)
    return w.view(np.uint32) if w.dtype == np.float32 else w


@pytest.mark.parametrize("kind", ["bf16", "fp16", "fp32", "fp8", "int8"])
def test_sequence_kernel_every_dtype(orc, kind):
    """A list of version-2 blobs of one container dtype runs as the sequence kernel; layers of assorted
    shapes (one tile up to several per CTA, ragged last tiles, r = 0 and r > 0) all match the oracle."""
    if kind == "fp8":
        comps = [ep.compress(synth.fp8_codes(64 + 16 * i, 512, seed=i), 5.0) for i in range(6)]
    elif kind == "int8":
        comps = [ep.compress(synth.int8_codes(64 + 8 * i, 256, seed=i), 3.0) for i in range(6)]
    else:
        comps = [ep.compress(synth.gaussian(8 + 37 * i % 300, 8 * (1 + i % 40), seed=i, container=kind), 2.0 + i % 6)
                 for i in range(12)]
        comps.append(ep.compress(synth.gaussian(200, 96, seed=99, container=kind), 9.0))  # raw low bits (r > 0)
    outs = [torch.empty(c.shape, dtype=c.dtype, device="cuda") for c in comps]
    for _ in range(2):
        ep.decompress_many(list(zip(comps, outs)))
    torch.cuda.synchronize()
    status_clean()
    for c, o in zip(comps, outs):
        assert np.array_equal(_bits_any(o), _want_any(orc, c))


def test_sequence_kernel_two_launch_groups(orc):
    """330 small layers: more than one sequence launch takes (280), so two groups run in stream order. Into
    separate outputs, then all into one buffer, where every element holds the last layer that wrote it."""
    comps = [ep.compress(synth.gaussian(1 + (i * 7) % 23, 8 * (1 + (i * 5) % 9), seed=2000 + i, container="bf16"),
                         1.0 + i % 9) for i in range(330)]
    outs = [torch.empty(c.shape, dtype=c.dtype, device="cuda") for c in comps]
    ep.decompress_many(list(zip(comps, outs)))
    torch.cuda.synchronize()
    status_clean()
    dec = [_want_any(orc, c) for c in comps]
    for d, o in zip(dec, outs):
        assert np.array_equal(gpu_bits(o), d)
    mx = max(c.shape[0] * c.shape[1] for c in comps)
    buf = torch.zeros(mx, dtype=torch.bfloat16, device="cuda")
    want = np.zeros(mx, np.uint16)
    for d in dec:
        want[: d.size] = d.reshape(-1)
    ep.decompress_many([(c, buf[: c.shape[0] * c.shape[1]].view(c.shape)) for c in comps])
    torch.cuda.synchronize()
    status_clean()
    assert np.array_equal(gpu_bits(buf), want)


@pytest.mark.parametrize("layout", ["one", "ping_pong", "offset"])
def test_sequence_kernel_overlapping_outputs(orc, layout):
    """Layers of mixed sizes (up to 14.7 M parameters) written into shared buffers: all into one, alternating
    between two, or into one at staggered offsets, so that a layer overwrites parts of several earlier ones.
    Each buffer must end as list-order decoding leaves it; run three times."""
    shapes = [(1024, 768), (96, 256), (768, 512), (64, 3840), (1536, 256), (256, 256), (1024, 640), (15360, 256),
              (3840, 3840), (2048, 512)]
    comps = [ep.compress(synth.dit_layer(60 + i, shape=s), 3.0 + 0.5 * (i % 3)) for i, s in enumerate(shapes)]
    dec = [_want_any(orc, c).reshape(-1) for c in comps]
    mx = max(M * N for M, N in shapes)
    bufs = [torch.zeros(mx + 4096, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    wants = [np.zeros(mx + 4096, np.uint16) for _ in range(2)]
    pairs = []
    for i, (c, (M, N)) in enumerate(zip(comps, shapes)):
        b = i % 2 if layout == "ping_pong" else 0
        off = (i * 1032) % 4096 // 8 * 8 if layout == "offset" else 0
        pairs.append((c, bufs[b][off: off + M * N].view(M, N)))
        wants[b][off: off + M * N] = dec[i]
    for _ in range(3):
        for b in bufs:
            b.zero_()
        ep.decompress_many(pairs)
        torch.cuda.synchronize()
        status_clean()
        for b, w in zip(bufs, wants):
            assert np.array_equal(gpu_bits(b), w)


@pytest.mark.parametrize("layout", ["separate", "one"])
def test_sequence_kernel_corrupt_blob_is_flagged_and_the_rest_decodes(orc, layout):
    """A corrupted word stream in one layer of a sequence: the sequence kernel flags it (EP_DEV_CORRUPT_TILE),
    every tile still publishes itself, so no wait runs out (no EP_DEV_DEP_WAIT) and the call completes; the
    other layers come out exact. With one shared buffer, the bytes the corrupt layer wrote last are the only
    ones left unspecified."""
    shapes = [(512, 512), (256, 768), (1024, 256), (384, 512)]
    comps = [ep.compress(synth.dit_layer(80 + i, shape=s), 4.0) for i, s in enumerate(shapes)]
    bad = bytearray(comps[1].blob)
    off_payload = int.from_bytes(bad[40:44], "little")
    for k in range(off_payload + 300, len(bad) - 64, 97):
        bad[k] ^= 0x5A
    comps[1] = ep.CompressedTensor(bytes(bad), comps[1].shape, comps[1].dtype, comps[1].actual_bpp)
    dec = {i: orc.decompress(c.blob).reshape(-1) for i, c in enumerate(comps) if i != 1}
    status_clean()
    if layout == "separate":
        outs = [torch.zeros(c.shape, dtype=c.dtype, device="cuda") for c in comps]
        ep.decompress_many(list(zip(comps, outs)))
        st = ep.device_status()
        assert st & 1 and not st & 16, st
        for i, o in enumerate(outs):
            if i != 1:
                assert np.array_equal(gpu_bits(o).reshape(-1), dec[i]), f"layer {i}"
    else:
        mx = max(M * N for M, N in shapes)
        buf = torch.zeros(mx, dtype=torch.bfloat16, device="cuda")
        ep.decompress_many([(c, buf[: c.shape[0] * c.shape[1]].view(c.shape)) for c in comps])
        st = ep.device_status()
        assert st & 1 and not st & 16, st
        got = gpu_bits(buf)
        last = np.full(mx, -1)
        for i, (M, N) in enumerate(shapes):
            last[: M * N] = i
        for i in dec:
            n = shapes[i][0] * shapes[i][1]
            sel = np.flatnonzero(last[:n] == i)
            assert np.array_equal(got[sel], dec[i][sel]), f"layer {i}"
    # the context stays usable
    good = ep.compress(synth.dit_layer(90, shape=(256, 256)), 4.0)
    assert np.array_equal(gpu_bits(ep.decompress(good)), orc.decompress(good.blob))
    status_clean()
