"""Per-layer bitrate plan (the README's mixed-bitrate packs): the oracle pinned, then the product's
ep_plan_bitrates held to it, then the plan's point checked on real blobs.

The oracle's pins are a general constrained solver on the same objective (scipy SLSQP), the closed
form of the unbounded case, the section sizes of blobs that the C oracle writes, and the tile-size
rule's worked cases. Each catches a different plausible slip: a wrong factor on log2(weight), a
dropped metadata term, a wrong section size, a wrong tile count.
"""
import math
import random

import numpy as np
import pytest
from scipy.optimize import minimize

import synth
from oracle import plan as oplan

DIT_SHAPES = [(3840, 3840), (10240, 3840), (3840, 10240), (15360, 256), (3840, 64), (64, 3840), (3840, 2560)]


def slsqp(shapes, weights, mean, lo_bound, hi_bound, rounds=0):
    """The same problem handed to a general solver: no KKT algebra, no water level."""
    n = np.array([r * c for r, c in shapes], float)
    meta = np.array([oplan.metadata_bits_per_param(r, c, rounds) for r, c in shapes])
    w = np.array(weights, float)
    tot = n.sum()
    f = lambda b: float((n * w * np.exp2(-2.0 * (b - meta))).sum() / tot)
    bounds = [(min(max(lo_bound, m), hi_bound), hi_bound) for m in meta]
    x0 = np.array([0.5 * (a + b) for a, b in bounds])
    res = minimize(f, x0, method="SLSQP", bounds=bounds,
                   constraints=[{"type": "eq", "fun": lambda b: float((n * b).sum() / tot - mean)}],
                   options={"ftol": 1e-14, "maxiter": 1000})
    # The solver may stop on its iteration limit close to the optimum: require a feasible point.
    assert abs(float((n * res.x).sum() / tot) - mean) < 1e-7, res.message
    assert all(a - 1e-9 <= v <= b + 1e-9 for v, (a, b) in zip(res.x, bounds))
    return res.x, f


@pytest.mark.parametrize("seed", range(8))
def test_oracle_plan_matches_general_solver(seed):
    rnd = random.Random(seed)
    k = rnd.randint(2, 6)
    shapes = [rnd.choice(DIT_SHAPES + [(256, 256), (512, 1024)]) for _ in range(k)]
    weights = [math.exp(rnd.gauss(0.0, 1.5)) for _ in range(k)]
    mean, lo, hi = rnd.uniform(1.0, 6.0), rnd.choice([0.001, 1.0]), rnd.choice([11.0, 7.0])
    b = oplan.plan(shapes, weights, mean, lo, hi)
    x, f = slsqp(shapes, weights, mean, lo, hi)
    assert f(np.array(b)) <= f(x) * (1 + 1e-9)          # no better point than the oracle's
    assert np.allclose(b, x, atol=2e-4)


def test_oracle_plan_closed_form_unbounded():
    # Equal shapes (equal metadata), no bound active: b_i = mean + log2(w_i / geometric mean of w) / 2.
    shapes = [(4096, 4096)] * 5
    w = [0.3, 1.0, 2.0, 7.5, 0.05]
    b = oplan.plan(shapes, w, 4.0)
    g = math.exp(sum(math.log(x) for x in w) / len(w))
    assert np.allclose(b, [4.0 + 0.5 * math.log2(x / g) for x in w], atol=1e-12)
    # Weights 1 and 16 are two bits apart.
    b2 = oplan.plan([(1024, 1024)] * 2, [1.0, 16.0], 3.0)
    assert abs((b2[1] - b2[0]) - 2.0) < 1e-12 and abs(sum(b2) - 6.0) < 1e-9


def test_oracle_plan_bounds_and_budget():
    shapes = [(4096, 4096), (4096, 4096), (64, 3840)]
    w = [1.0, 1e-6, 1.0]
    b = oplan.plan(shapes, w, 2.0, min_bpp=1.0, max_bpp=11.0)
    assert b[1] == 1.0                                  # a layer nobody cares about sits at its floor
    meta = oplan.metadata_bits_per_param(64, 3840)
    # equal weights: the two free layers share the water level, each above its own metadata
    assert abs((b[2] - meta) - (b[0] - oplan.metadata_bits_per_param(4096, 4096))) < 1e-9
    n = [r * c for r, c in shapes]
    assert abs(sum(x * y for x, y in zip(n, b)) / sum(n) - 2.0) < 1e-9
    # Budgets out of reach: every layer at its floor, or at the ceiling.
    assert oplan.plan(shapes, w, 0.001, min_bpp=0.001) == [oplan.metadata_bits_per_param(r, c) for r, c in shapes]
    assert oplan.plan(shapes, w, 5.0, max_bpp=5.0) == [5.0] * 3


def test_oracle_auto_rounds_worked_cases():
    wave = 148 * 32
    assert oplan.auto_rounds(256 * 256 // 8) == 16                    # far below half a wave
    assert oplan.auto_rounds(512 * (wave // 2) - 512) == 16           # one tile short of half a wave
    assert oplan.auto_rounds(512 * wave) == 16                        # exactly one wave of 16-round tiles
    # 3600 tiles of 16 = 0.76 wave -> 1 wave: G = ceil(1843200 / (32 * 4736)) = ceil(12.16) = 13
    assert oplan.auto_rounds(3840 * 3840 // 8) == 13
    # 9600 tiles of 16 = 2.03 waves -> 2 waves: G = ceil(4915200 / (32 * 4736 * 2)) = ceil(16.22) = 17
    assert oplan.auto_rounds(10240 * 3840 // 8) == 17
    # 57344 tiles of 16 = 12.11 waves -> 12 waves: G = ceil(29360128 / (32 * 4736 * 12)) = ceil(16.14) = 17
    assert oplan.auto_rounds(8192 * 28672 // 8) == 17
    # 1.8 waves of 16 -> floor(1.8 + 0.25) = 2 waves: G = ceil(4364697 / (32 * 4736 * 2)) = ceil(14.4) = 15
    assert oplan.auto_rounds(int(1.8 * 512 * wave)) == 15
    # exactly half a wave of 16 -> 1 wave: ceil(1212416 / (32 * 4736)) = 8, raised to the floor of 12
    assert oplan.auto_rounds(512 * (wave // 2)) == 12


@pytest.mark.parametrize("version", [1, 2])
@pytest.mark.parametrize("shape,G", [((256, 256), 16), ((129, 8), 2), ((300, 64), 5), ((64, 3840), 16)])
def test_oracle_metadata_matches_written_blobs(orc, shape, G, version):
    # The fixed sections of a blob the C oracle writes, with its tables section swapped for the largest
    # (640 frequencies of 12 bits in version 1, 8 bits in version 2).
    M, N = shape
    w = synth.gaussian(M, N, seed=M + N, container="bf16")
    blob, _ = orc.compress(synth.container_bits(w), synth.dtype_code(w), 3.0, G,
                           prob_bits=12 if version == 1 else 8)
    hdr = np.frombuffer(blob[:64], np.uint8)
    u32 = lambda off: int(hdr[off:off + 4].view(np.uint32)[0])
    T, off_tables, off_offsets, off_payload = u32(24), u32(32), u32(36), u32(40)
    largest = 18 + (960 if version == 1 else 640)
    fixed = off_payload - (off_offsets - off_tables) + oplan.pad16(largest)
    assert abs(oplan.metadata_bits_per_param(M, N, G, version) - 8.0 * (fixed + 104 * T) / (M * N)) < 1e-12


# --- product parity -----------------------------------------------------------------------------

@pytest.fixture(scope="module")
def ep():
    import decode_ep_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("seed", range(40))
def test_plan_bitrates_matches_oracle(ep, seed):
    rnd = random.Random(100 + seed)
    k = rnd.randint(1, 300)
    shapes = [(rnd.randint(1, 16384), 8 * rnd.randint(1, 2048)) for _ in range(k)]
    weights = [math.exp(rnd.gauss(0.0, rnd.choice([0.1, 1.0, 4.0]))) for _ in range(k)]
    lo = rnd.choice([0.001, 0.5, 2.0])
    hi = rnd.choice([11.0, 6.0, max(lo, 3.0)])
    mean = rnd.uniform(0.001, hi)
    G = rnd.choice([0, 0, 7, 16])
    got = ep.plan_bitrates(shapes, weights, mean, lo, hi, rounds_per_tile=G)
    want = oplan.plan(shapes, weights, mean, lo, hi, rounds=G)
    assert np.allclose(got, want, rtol=0, atol=1e-9)


def test_plan_bitrates_dit_set(ep):
    shapes = [(M, N) for _, M, N in synth.dit_layer_shapes()]
    rnd = random.Random(5)
    weights = [math.exp(rnd.gauss(0.0, 1.0)) for _ in shapes]
    got = ep.plan_bitrates(shapes, weights, 2.3)
    assert np.allclose(got, oplan.plan(shapes, weights, 2.3), rtol=0, atol=1e-9)
    n = np.array([M * N for M, N in shapes], float)
    assert abs(float((n * np.array(got)).sum() / n.sum()) - 2.3) < 1e-9


def test_plan_bitrates_errors(ep):
    with pytest.raises(ep.EntroPackError) as e:
        ep.plan_bitrates([(16, 16)], [0.0], 2.0)
    assert e.value.status == -1
    with pytest.raises(ep.EntroPackError) as e:
        ep.plan_bitrates([(16, 12)], [1.0], 2.0)
    assert e.value.status == -3
    for bad in [dict(mean_bpp=12.0), dict(mean_bpp=2.0, min_bpp=3.0, max_bpp=2.5), dict(mean_bpp=5.0, max_bpp=4.0),
                dict(mean_bpp=float("nan"))]:
        with pytest.raises(ep.EntroPackError) as e:
            ep.plan_bitrates([(16, 16)], [1.0], **bad)
        assert e.value.status == -4
    with pytest.raises(ep.EntroPackError):
        ep.plan_bitrates([(16, 16)], [1.0, 2.0], 2.0)


# --- the point of the plan, on blobs ---------------------------------------------------------------

def test_mixed_plan_lowers_weighted_error_at_equal_storage(orc):
    """Layers of unequal sensitivity, compressed and decoded by the oracle: at the same total storage,
    the planned targets give a lower sensitivity-weighted squared error than one uniform target."""
    shapes = [(128, 512)] * 4 + [(256, 256)] * 4
    rnd = random.Random(11)
    sens = [math.exp(rnd.gauss(0.0, 1.0)) for _ in shapes]
    ws = [synth.gaussian(M, N, seed=40 + i, std=0.02 * math.exp(0.3 * rnd.gauss(0.0, 1.0)), container="bf16")
          for i, (M, N) in enumerate(shapes)]
    ref = [w.float().numpy().astype(np.float64) for w in ws]
    weights = [s * float((r * r).mean()) for s, r in zip(sens, ref)]

    def run(targets):
        bits, cost = 0, 0.0
        for w, r, s, t in zip(ws, ref, sens, targets):
            blob, _ = orc.compress(synth.container_bits(w), synth.dtype_code(w), t, 16)
            y = orc.decompress(blob).view(np.uint16).astype(np.uint32) << 16
            d = y.view(np.float32).astype(np.float64) - r
            bits += 8 * len(blob)
            cost += s * float((d * d).sum())
        return bits, cost

    mean = 2.3
    planned = oplan.plan(shapes, weights, mean, rounds=16)
    bits_u, cost_u = run([mean] * len(shapes))
    bits_m, cost_m = run(planned)
    assert bits_m <= bits_u * 1.01
    assert cost_m < 0.8 * cost_u
