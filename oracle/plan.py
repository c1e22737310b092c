"""Oracle for the per-layer bitrate plan: which target each layer of a set gets under one budget.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite may import this module. It shares no code
with the product library (``decode_ep_b200``) and imports nothing from it.

Source: the EntroPack README (``README_zh.md``, section "Pre-quantised models") describes packs of
"extreme mixed bitrate", whose bits are allocated per layer by sensitivity (2.3 bpp on Z-Image-Turbo,
3.0 bpp on the other two models). The pages give no rule; the reading taken here is the textbook
high-rate allocation. A layer coded at R data bits per parameter has a squared error proportional to
2^(-2R); layer i of n_i parameters costs weight_i per unit of that error; its blob spends meta_i bits
per parameter on metadata, which buys no accuracy. Minimise

    sum_i n_i * weight_i * 2^(-2 (b_i - meta_i))
    subject to  sum_i n_i * b_i = mean_bpp * sum_i n_i,   max(min_bpp, meta_i) <= b_i <= max_bpp.

Setting the derivative of the Lagrangian to zero for each free b_i gives
    b_i = meta_i + log2(weight_i)/2 + theta
with one theta for every layer; bound layers sit at their bound. The oracle finds theta by plain
bisection on the budget (which rises with theta), 200 halvings in double precision.

meta_i is written out from the EPK1 format description: a 64-byte header, bf16 row scales padded to
16 bytes, the largest tables section (18 bytes of context ranges and one frequency for each of the 640
symbols, 8 bits in format version 2 and 12 in version 1, padded), the (T+1) u32 tile offsets padded, and
the storage estimate's 104 bytes per tile for the final rANS states. T = ceil(groups / (32 G)), with the
format's automatic tile size G.

Parity pins: ``tests/test_plan.py`` checks this against a general constrained solver
(scipy's SLSQP) on the same objective, the closed form of the unbounded case, and the section sizes
of blobs the C oracle writes.
"""
from __future__ import annotations

import math

HEADER_BYTES = 64
MAX_TABLE_SYMBOLS = 128 + 8 * 64
SMS, WARPS_PER_SM = 148, 32


def pad16(n: int) -> int:
    return (n + 15) // 16 * 16


def auto_rounds(groups: int) -> int:
    """The format's tile size: 16 rounds, unless the tensor has at least half a wave of 16-round
    tiles (a wave = 148 SMs x 32 warps); then the G in [12, 24] whose tiles fill whole waves."""
    slots = SMS * WARPS_PER_SM
    tiles16 = math.ceil(groups / 512)
    if tiles16 < slots / 2:
        return 16
    waves = max(1, math.floor(tiles16 / slots + 0.25))
    return int(min(24, max(12, math.ceil(groups / (32 * slots * waves)))))


def metadata_bits_per_param(rows: int, cols: int, rounds: int = 0, version: int = 2) -> float:
    groups = rows * cols // 8
    G = rounds if rounds else auto_rounds(groups)
    tiles = -(-groups // (32 * G))
    fbits = 12 if version == 1 else 8
    tables = 2 * 9 + -(-fbits * MAX_TABLE_SYMBOLS // 8)
    meta = HEADER_BYTES + pad16(2 * rows) + pad16(tables) + pad16(4 * (tiles + 1)) + 104 * tiles
    return 8.0 * meta / (rows * cols)


def plan(shapes, weights, mean_bpp, min_bpp=0.001, max_bpp=11.0, rounds=0, version=2):
    """Per-layer targets b_i (list of floats) for layers of the given (rows, cols) shapes."""
    n = [r * c for r, c in shapes]
    meta = [metadata_bits_per_param(r, c, rounds, version) for r, c in shapes]
    lo = [min(max(min_bpp, m), max_bpp) for m in meta]
    hi = [max_bpp] * len(shapes)
    free = [m + 0.5 * math.log2(w) for m, w in zip(meta, weights)]

    def rates(theta):
        return [min(h, max(l, f + theta)) for f, l, h in zip(free, lo, hi)]

    def spent(theta):
        return sum(ni * bi for ni, bi in zip(n, rates(theta)))

    budget = mean_bpp * sum(n)
    if budget <= sum(ni * li for ni, li in zip(n, lo)):
        return lo
    if budget >= sum(ni * hi_ for ni, hi_ in zip(n, hi)):
        return hi
    a = min(l - f for l, f in zip(lo, free)) - 1.0
    b = max(h - f for h, f in zip(hi, free)) + 1.0
    for _ in range(200):
        mid = 0.5 * (a + b)
        if spent(mid) < budget:
            a = mid
        else:
            b = mid
    return rates(0.5 * (a + b))


def objective(shapes, weights, bpp, rounds=0, version=2):
    """The quantity the plan minimises, for any assignment of targets."""
    return sum(r * c * w * 2.0 ** (-2.0 * (b - metadata_bits_per_param(r, c, rounds, version)))
               for (r, c), w, b in zip(shapes, weights, bpp))
