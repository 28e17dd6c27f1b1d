"""Pins for the oracle's online N:M mask and its metadata encoding.

The oracle ranks by a count of "beating" elements; the references here sort,
which is a different algorithm for the same definition (top-N by magnitude per
group of M, ties to the lower index; the 4:8 pair pattern keeps the top 2 of 4
adjacent pairs scored by their larger magnitude).
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sort_keep(group, n):
    order = sorted(range(len(group)), key=lambda i: (-abs(group[i]), i))
    keep = np.zeros(len(group), np.uint8)
    keep[order[:n]] = 1
    return keep


def _sort_keep_pairs(group):
    scores = [max(abs(group[2 * p]), abs(group[2 * p + 1])) for p in range(4)]
    order = sorted(range(4), key=lambda p: (-scores[p], p))
    keep = np.zeros(8, np.uint8)
    for p in order[:2]:
        keep[2 * p] = keep[2 * p + 1] = 1
    return keep


def _rows_of_groups(groups, m):
    g = np.asarray(groups, np.float32).reshape(-1, m)
    # pad each row to a multiple of 256 so the oracle's row length rule holds
    per_row = 256 // m
    nrows = (g.shape[0] + per_row - 1) // per_row
    pad = np.zeros((nrows * per_row - g.shape[0], m), np.float32)
    return np.concatenate([g, pad]).reshape(nrows, 256), g.shape[0]


def test_2_4_exhaustive_small_integers():
    vals = [-2.0, -1.0, 0.0, 1.0, 2.0]
    groups = list(itertools.product(vals, repeat=4))
    x, ng = _rows_of_groups(groups, 4)
    keep = oracle.mask(x, "2:4").reshape(-1, 4)[:ng]
    for g, k in zip(groups, keep):
        np.testing.assert_array_equal(k, _sort_keep(g, 2), err_msg=str(g))


def test_4_8_pair_exhaustive_small_integers():
    rng = np.random.default_rng(5)
    groups = [np.array(t) * rng.choice([-1.0, 1.0], 8) for t in itertools.product([0.0, 1.0, 2.0], repeat=8)]
    x, ng = _rows_of_groups(groups, 8)
    keep = oracle.mask(x, "4:8pair").reshape(-1, 8)[:ng]
    for g, k in zip(groups, keep):
        np.testing.assert_array_equal(k, _sort_keep_pairs(list(g)), err_msg=str(g))


def test_8_16_random_and_adversarial_ties():
    rng = np.random.default_rng(6)
    groups = [rng.integers(-3, 4, 16).astype(np.float64) for _ in range(3000)]
    groups += [np.full(16, 1.0), np.zeros(16), np.where(np.arange(16) % 2 == 0, 5.0, -5.0)]
    groups += [rng.standard_normal(16) for _ in range(500)]
    x, ng = _rows_of_groups(groups, 16)
    keep = oracle.mask(x, "8:16").reshape(-1, 16)[:ng]
    for g, k in zip(groups, keep):
        np.testing.assert_array_equal(k, _sort_keep(list(np.float32(g)), 8))


@pytest.mark.parametrize("pat,m", [("2:4", 4), ("4:8pair", 8), ("8:16", 16), ("8:16pair", 16)])
def test_exactly_half_kept_and_pruning_ratio(pat, m):
    # Huawei problem 137-2, "模块六": pruning ratio R = pruned / total; every
    # pattern keeps N = M/2, so R is exactly 50% (the problem's target).
    rng = np.random.default_rng(7)
    x = rng.standard_t(3, size=(64, 1024)).astype(np.float32)
    x[:, ::7] = 0.0  # zeros and ties
    keep = oracle.mask(x, pat)
    per_group = keep.reshape(64, -1, m).sum(axis=2)
    assert np.all(per_group == m // 2)
    assert (keep == 0).sum() / keep.size == 0.5


def test_group_maximum_is_always_kept():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((32, 512)) * np.exp(rng.uniform(-3, 3, (32, 512)))).astype(np.float32)
    for pat, m in (("2:4", 4), ("4:8pair", 8), ("8:16", 16)):
        keep = oracle.mask(x, pat).reshape(-1, m)
        a = np.abs(x).reshape(-1, m)
        top = np.argmax(a, axis=1)  # first index of the maximum
        assert np.all(keep[np.arange(a.shape[0]), top] == 1), pat


def _golden_cost():
    out = {}
    with open(os.path.join(GOLDEN, "metadata_cost.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                p, v = line.split()
                out[p] = float(v)
    return out


@pytest.mark.parametrize("pat,m,n", [("2:4", 4, 2), ("8:16", 16, 8)])
def test_mask_space_matches_published_metadata_cost(pat, m, n):
    """Every N-of-M subset is reachable, so one group's mask carries log2 C(M,N)
    bits; rounded up per group this is the 8:16 page's 0.75 / 0.875 bit/elem."""
    rng = np.random.default_rng(9)
    seen = set()
    if m == 4:
        for t in itertools.permutations(range(1, 5)):
            x, _ = _rows_of_groups([t], 4)
            seen.add(tuple(oracle.mask(x, pat)[0, :4]))
    else:
        # one group per 8-subset: magnitudes 2 on the subset, 1 elsewhere (random signs)
        groups = []
        for sub in itertools.combinations(range(16), 8):
            g = np.ones(16) * rng.choice([-1.0, 1.0], 16)
            g[list(sub)] *= 2.0
            groups.append(g)
        x, ng = _rows_of_groups(groups, 16)
        for k in oracle.mask(x, pat).reshape(-1, 16)[:ng]:
            seen.add(tuple(k))
    assert len(seen) == math.comb(m, n)
    assert math.ceil(math.log2(len(seen))) / m == _golden_cost()[pat]


def _decode_meta_ref(meta_row, k, pat):
    keep = np.zeros(k, np.uint8)
    if pat == "8:16":
        for g in range(k // 16):
            mask = int(meta_row[2 * g]) | (int(meta_row[2 * g + 1]) << 8)
            keep[16 * g:16 * g + 16] = [(mask >> j) & 1 for j in range(16)]
        return keep
    unit = 2 if pat == "4:8pair" else 1
    for g in range(k // (4 * unit)):
        nib = (int(meta_row[g // 2]) >> (4 * (g % 2))) & 15
        i0, i1 = nib & 3, nib >> 2
        assert i0 < i1, "kept indices must be ascending"
        for u in range(unit):
            keep[g * 4 * unit + i0 * unit + u] = 1
            keep[g * 4 * unit + i1 * unit + u] = 1
    return keep


@pytest.mark.parametrize("pat", ["2:4", "4:8pair", "8:16"])
def test_metadata_encodes_the_mask(pat):
    rng = np.random.default_rng(10)
    x = rng.standard_normal((8, 512)).astype(np.float32)
    prep = oracle.prepare(x, "mxfp4", pat)
    keep = oracle.mask(x, pat)
    for r in range(8):
        np.testing.assert_array_equal(_decode_meta_ref(prep["meta"][r], 512, pat), keep[r])


# ------------------------------------------------ 8:16 re-packed (4:8 pair layout)
def _sort_keep_repacked(group16):
    """The re-packed rule by sorting: top 8 of the 16 (ties to the lower index),
    then per half the 2 pairs ranked by (count of those 8 they hold, larger
    magnitude, lower index first)."""
    k16 = _sort_keep(group16, 8)
    keep = np.zeros(16, np.uint8)
    for half in range(2):
        base = 8 * half
        key = []
        for p in range(4):
            a, b = base + 2 * p, base + 2 * p + 1
            key.append((-(int(k16[a]) + int(k16[b])), -max(abs(group16[a]), abs(group16[b])), p))
        for _, _, p in sorted(key)[:2]:
            keep[base + 2 * p] = keep[base + 2 * p + 1] = 1
    return keep


def test_8_16_pair_against_sorting_with_ties():
    rng = np.random.default_rng(16)
    groups = [rng.integers(-3, 4, 16).astype(np.float64) for _ in range(3000)]
    groups += [np.full(16, 1.0), np.zeros(16), np.where(np.arange(16) % 2 == 0, 5.0, -5.0)]
    groups += [rng.standard_normal(16) for _ in range(500)]
    x, ng = _rows_of_groups(groups, 16)
    keep = oracle.mask(x, "8:16pair").reshape(-1, 16)[:ng]
    for g, k in zip(groups, keep):
        np.testing.assert_array_equal(k, _sort_keep_repacked(list(np.float32(g))), err_msg=str(g))


def test_8_16_pair_is_a_4_8_pair_mask():
    rng = np.random.default_rng(17)
    x = rng.standard_t(3, size=(32, 1024)).astype(np.float32)
    x[:, ::5] = 0.0
    keep = oracle.mask(x, "8:16pair").reshape(32, -1, 4, 2)
    assert np.all(keep[..., 0] == keep[..., 1])           # whole pairs
    assert np.all(keep[..., 0].sum(axis=-1) == 2)         # two of four per group of 8


def test_8_16_pair_equals_8_16_where_the_selection_fits():
    """When the top 8 of every 16 already sit in two whole pairs of each half,
    the re-packed mask IS the 8:16 mask (nothing overflows into the residual)."""
    rng = np.random.default_rng(18)
    x = (rng.random((16, 512)).astype(np.float32) * 0.5).reshape(16, -1, 2, 4, 2)  # small everywhere
    for r in range(16):
        for g in range(x.shape[1]):
            for h in range(2):
                p0, p1 = rng.choice(4, 2, replace=False)
                x[r, g, h, [p0, p1], :] = rng.uniform(1.0, 8.0, (2, 2)) * rng.choice([-1, 1], (2, 2))
    x = x.reshape(16, 512)
    np.testing.assert_array_equal(oracle.mask(x, "8:16pair"), oracle.mask(x, "8:16"))


def test_8_16_pair_metadata_is_the_4_8_pair_encoding():
    rng = np.random.default_rng(19)
    x = rng.standard_normal((4, 256)).astype(np.float32)
    prep = oracle.prepare(x, "mxfp4", "8:16pair")
    keep = oracle.mask(x, "8:16pair")
    assert prep["meta"].shape == (4, 256 // 16) and prep["bb_codes"].shape == (4, 256 // 4)
    for r in range(4):
        for g in range(256 // 8):
            nib = (prep["meta"][r, g // 2] >> (4 * (g % 2))) & 15
            kept = [p for p in range(4) if keep[r, 8 * g + 2 * p]]
            assert nib == (kept[0] | (kept[1] << 2))
