"""CUDA encoder parity: ep_compress_cuda must write the same blob bytes as the oracle encoder and the host
encoder.

The CUDA encoder and the host encoder compile the same lattice and table code, so agreement between those
two alone would not check that code. Every case is therefore also compared, byte for byte, with the
oracle's encoder (oracle/, which shares no code with either) on the same input, the oracle taking the
tile size G from the product blob's header. Integer and byte work is held to bit-exactness: every scale,
every bisection decision, every lattice point and every rANS word must agree.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ep():
    import decode_ep_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


CASES = [
    ("quickstart", lambda: synth.quickstart_256(), 3.5, 16),
    ("outliers_esc", lambda: synth.lognormal_rows_with_outliers(n=256, seed=11, outlier_frac=2e-3, outlier_mult=40.0), 4.0, 16),
    ("fp16_raw_bits", lambda: synth.gaussian(128, 128, seed=8, container="fp16"), 9.0, 16),
    ("ragged_1_group_tile", lambda: synth.gaussian(129, 8, seed=3, container="bf16"), 3.0, 2),
    ("fp8", lambda: synth.fp8_codes(64, 512, seed=3), 5.0, 16),
    ("int8", lambda: synth.int8_codes(64, 512, seed=4), 3.0, 16),
    ("fp32_11bpp", lambda: synth.gaussian(96, 64, seed=5, container="fp32"), 11.0, 16),
    ("all_zero", lambda: torch.zeros(64, 64, dtype=torch.bfloat16), 2.0, 16),
    ("below_floor", lambda: synth.gaussian(64, 64, seed=3, container="bf16"), 0.001, 16),
    ("dit_like", lambda: synth.dit_layer(3, shape=(512, 256)), 4.0, 16),
    ("G1024", lambda: synth.gaussian(200, 96, seed=9, container="bf16"), 2.5, 1024),
    ("one_row", lambda: synth.gaussian(1, 4096, seed=13, container="bf16"), 4.0, 0),
    ("r12_extreme", lambda: synth.gaussian(64, 64, seed=14, container="fp32"), 11.0, 3),
    ("zero_rows", lambda: torch.cat([torch.zeros(3, 64), synth.gaussian(5, 64, seed=15)]).to(torch.bfloat16), 4.0, 1),
]


VERSIONS = [2, 1]


def both(ep, w, cfg_kwargs):
    host = ep.compress(w, ep.EntroPackLossyConfig(**cfg_kwargs))
    dev = ep.compress(w.cuda(), ep.EntroPackLossyConfig(encoder="cuda", **cfg_kwargs))
    return host, dev


def oracle_bytes(orc, w, target, blob):
    """The oracle encoder's blob for the same input and target, at the tile size G and format version the
    product chose."""
    G = int.from_bytes(blob[20:22], "little")
    version = int.from_bytes(blob[4:6], "little")
    ob, _ = orc.compress(synth.container_bits(w.cpu()), synth.dtype_code(w), target, G,
                         prob_bits=12 if version == 1 else 8)
    return ob


@pytest.mark.parametrize("version", VERSIONS)
@pytest.mark.parametrize("name,maker,target,G", CASES, ids=[c[0] for c in CASES])
def test_cuda_encoder_matches_oracle_and_host_bytes(ep, orc, name, maker, target, G, version):
    w = maker()
    host, dev = both(ep, w, dict(target_bpp=target, rounds_per_tile=G, format_version=version))
    assert dev.blob == oracle_bytes(orc, w, target, dev.blob), "CUDA encoder differs from the oracle encoder"
    assert dev.blob == host.blob
    assert dev.actual_bpp == host.actual_bpp


@pytest.mark.parametrize("version", VERSIONS)
@pytest.mark.parametrize("workload", ["lognormal3072", "dit_q_3840"])
def test_cuda_encoder_matches_oracle_full_size(ep, orc, workload, version):
    """Full-size tensors against the oracle encoder directly: the 3072x3072 lognormal-rows matrix with
    outliers and one 3840x3840 layer of the DiT-like set, both at 4 bpp."""
    w = synth.lognormal_rows_with_outliers() if workload == "lognormal3072" else synth.dit_layer(0)
    dev = ep.compress(w.cuda(), ep.EntroPackLossyConfig(4.0, encoder="cuda", format_version=version))
    assert dev.blob == oracle_bytes(orc, w, 4.0, dev.blob)


@pytest.mark.parametrize("workload", ["lognormal3072", "dit_gate", "fp8_rows", "sweep_6bpp"])
def test_cuda_encoder_full_size_workloads(ep, workload):
    # Full-size shapes of the benchmark configs (the FP8 one cut to 1024 rows to keep the test short).
    if workload == "lognormal3072":
        w, t = synth.lognormal_rows_with_outliers(), 4.0
    elif workload == "dit_gate":
        w, t = synth.dit_layer(4), 4.0
    elif workload == "fp8_rows":
        w, t = synth.fp8_codes(1024, 28672, seed=3), 5.0
    else:
        w, t = synth.gaussian(4096, 4096, 2, container="bf16"), 6.0
    host, dev = both(ep, w, dict(target_bpp=t))
    assert dev.blob == host.blob


def test_cuda_encoder_strided_input_and_decode(ep):
    base = synth.gaussian(64, 96, seed=12, container="bf16").cuda()
    view = base[:, 16:80]
    a = ep.compress(view, ep.EntroPackLossyConfig(3.0, encoder="cuda"))
    b = ep.compress(view.cpu().contiguous(), 3.0)
    assert a.blob == b.blob
    y = ep.decompress(a)
    assert y.shape == (64, 64) and torch.isfinite(y.float()).all()


def test_cuda_encoder_errors(ep):
    w = synth.gaussian(16, 16, seed=1, container="bf16").cuda()
    with pytest.raises(ep.EntroPackError) as e:
        ep.compress(w, ep.EntroPackLossyConfig(11.5, encoder="cuda"))
    assert e.value.status == -4
    x = torch.zeros(8, 16, device="cuda")
    x[3, 3] = float("nan")
    with pytest.raises(ep.EntroPackError) as e:
        ep.compress(x, ep.EntroPackLossyConfig(3.0, encoder="cuda"))
    assert e.value.status == -5
    with pytest.raises(ep.EntroPackError) as e:
        ep.compress(w.cpu(), ep.EntroPackLossyConfig(3.0, encoder="cuda"))
    assert e.value.status == -1


@pytest.mark.parametrize("version", VERSIONS)
@pytest.mark.parametrize("seed", range(16))
def test_cuda_encoder_matches_oracle_and_host_bytes_fuzz(ep, orc, seed, version):
    import random
    rnd = random.Random(2000 + seed)
    M, N = rnd.randint(1, 200), 8 * rnd.randint(1, 64)
    kind = rnd.choice(["bf16", "fp16", "fp32", "fp8", "int8"])
    if kind == "fp8":
        w = synth.fp8_codes(M, N, seed=seed)
    elif kind == "int8":
        w = synth.int8_codes(M, N, seed=seed)
    else:
        w = synth.gaussian(M, N, seed=seed, std=rnd.choice([0.02, 1.0, 300.0]), container=kind)
    cfg = dict(target_bpp=round(rnd.uniform(0.3, 11.0), 3), rounds_per_tile=rnd.choice([0, 1, 3, 16, 33]),
               format_version=version)
    host, dev = both(ep, w, cfg)
    assert dev.blob == host.blob
    assert dev.blob == oracle_bytes(orc, w, cfg["target_bpp"], dev.blob)
