"""Pins for the oracle's number formats (E2M1, E4M3, E8M0, exact floor-log2).

Each check compares the oracle with something other than itself: the OCP
tables in tests/golden, a brute-force nearest-value search written here in
fp64, and CUDA's host-side conversion functions (cuda_fp4.h / cuda_fp8.h).
"""
import ctypes
import math
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


def _golden_pairs(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                a, b = line.split()
                rows.append((a, b))
    return rows


@pytest.fixture(scope="module")
def cuconv():
    """CUDA's host conversion functions, compiled from tests/helpers (needs nvcc)."""
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = os.path.join(HERE, "helpers", "cuda_host_convert.cu")
    bdir = os.path.join(HERE, "helpers", "_build")
    os.makedirs(bdir, exist_ok=True)
    lib = os.path.join(bdir, "cuda_host_convert.so")
    if not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
        tmp = lib + f".{os.getpid()}.tmp"
        subprocess.run([nvcc, "-O1", "-Wno-deprecated-gpu-targets", "-Xcompiler", "-fPIC", "-shared", "-o", tmp,
                        src], check=True)
        os.replace(tmp, lib)
    return ctypes.CDLL(lib)


def _cu_call(lib, name, inp, out_dtype):
    inp = np.ascontiguousarray(inp)
    out = np.zeros(inp.size, out_dtype)
    getattr(lib, name)(ctypes.c_void_p(inp.ctypes.data), ctypes.c_int64(inp.size), ctypes.c_void_p(out.ctypes.data))
    return out


E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _brute_e2m1(v):
    """Nearest E2M1 magnitude in fp64, ties to the even code, saturating, sign kept."""
    out = np.zeros(v.size, np.uint8)
    for i, x in enumerate(v.astype(np.float64)):
        a = min(abs(x), 6.0)  # satfinite: everything past the largest magnitude maps to it
        d = np.abs(E2M1_GRID - a)
        best = np.flatnonzero(d == d.min())
        c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out[i] = c | (8 if math.copysign(1.0, x) < 0 else 0)
    return out


def _e2m1_probe_values():
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 8.0], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(np.inf))])
    rng = np.random.default_rng(1)
    rand = (rng.standard_normal(4000) * 3).astype(np.float32)
    tiny = np.array([0.0, 1e-45, 1e-30, 0.1, 100.0, 3.4e38], np.float32)
    v = np.concatenate([near, rand, tiny, E2M1_GRID.astype(np.float32)])
    return np.concatenate([v, -v]).astype(np.float32)


def test_e2m1_decode_matches_ocp_table():
    for code, val in _golden_pairs("e2m1_grid.txt"):
        got = oracle.e2m1_decode([int(code)])[0]
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code


def test_e2m1_encode_brute_force():
    v = _e2m1_probe_values()
    np.testing.assert_array_equal(oracle.e2m1_encode(v), _brute_e2m1(v))


def test_e2m1_encode_every_midpoint_rounds_to_even():
    # midpoints between neighbouring grid values go to the neighbour with the even code
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for m, c in expect.items():
        assert oracle.e2m1_encode([m])[0] == c
        assert oracle.e2m1_encode([-m])[0] == c | 8


def test_e2m1_encode_matches_cuda_host(cuconv):
    v = _e2m1_probe_values()
    np.testing.assert_array_equal(oracle.e2m1_encode(v), _cu_call(cuconv, "cu_e2m1_encode_n", v, np.uint8))


def test_e2m1_roundtrip_all_codes(cuconv):
    codes = np.arange(16, dtype=np.uint8)
    vals = oracle.e2m1_decode(codes)
    np.testing.assert_array_equal(vals, _cu_call(cuconv, "cu_e2m1_decode_n", codes, np.float32))
    np.testing.assert_array_equal(oracle.e2m1_encode(vals), codes)


def _e4m3_ref_decode(c):
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    if e == 15 and m == 7:
        return math.nan
    v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -v if s else v


def test_e4m3_decode_all_codes(cuconv):
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = np.array([_e4m3_ref_decode(int(c)) for c in codes])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok].astype(np.float32))
    cu = _cu_call(cuconv, "cu_e4m3_decode_n", codes, np.float32)
    np.testing.assert_array_equal(got[ok], cu[ok])
    for code, val in _golden_pairs("e4m3_anchors.txt"):
        assert oracle.e4m3_decode([int(code, 16)])[0] == float(val)


def _e4m3_probe_values():
    finite = np.array([_e4m3_ref_decode(c) for c in range(127)], np.float64)
    mids = ((finite[:-1] + finite[1:]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(np.inf))])
    rng = np.random.default_rng(2)
    rand = np.exp(rng.uniform(-16, 7, 5000)).astype(np.float32)
    big = np.array([448.0, 449.0, 464.0, 465.0, 480.0, 1e6, 3.4e38], np.float32)
    v = np.concatenate([near, rand, big, finite.astype(np.float32), [0.0, 1e-45]]).astype(np.float32)
    return np.concatenate([v, -v])


def test_e4m3_encode_brute_force():
    finite = np.array([_e4m3_ref_decode(c) for c in range(127)], np.float64)
    v = _e4m3_probe_values()
    got = oracle.e4m3_encode(v)
    for x, g in zip(v.astype(np.float64), got):
        a = min(abs(x), 448.0)  # satfinite
        d = np.abs(finite - a)
        best = np.flatnonzero(d == d.min())
        c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        c |= 0x80 if math.copysign(1, x) < 0 else 0
        assert g == c, (x, g, c)


def test_e4m3_encode_matches_cuda_host(cuconv):
    v = _e4m3_probe_values()
    np.testing.assert_array_equal(oracle.e4m3_encode(v), _cu_call(cuconv, "cu_e4m3_encode_n", v, np.uint8))


def test_e8m0_decode_is_power_of_two():
    codes = np.arange(255, dtype=np.uint8)
    got = oracle.e8m0_decode(codes)
    ref = np.array([math.ldexp(1.0, int(c) - 127) for c in codes], np.float32)
    np.testing.assert_array_equal(got, ref)


def test_floor_log2_exact_including_subnormals():
    rng = np.random.default_rng(3)
    pw = np.array([math.ldexp(1.0, e) for e in range(-149, 128)], np.float32)
    v = np.concatenate([pw, np.nextafter(pw, np.float32(0))[1:], np.nextafter(pw, np.float32(np.inf))[:-1],
                        np.exp(rng.uniform(-100, 80, 3000)).astype(np.float32)])
    v = v[(v > 0) & np.isfinite(v)]
    ref = np.array([math.frexp(float(x))[1] - 1 for x in v], np.int32)
    np.testing.assert_array_equal(oracle.floor_log2(v), ref)


def test_tensor_scale_closed_form():
    # g_enc = 6 * 448 / amax and its inverse; amax = 0 leaves the scale at 1
    ge, gd = oracle.tensor_scale(2688.0)
    assert ge == 1.0 and gd == 1.0
    ge, gd = oracle.tensor_scale(168.0)  # 2688 / 16
    assert ge == 16.0 and gd == 1.0 / 16
    assert oracle.tensor_scale(0.0) == (1.0, 1.0)
    ge, gd = oracle.tensor_scale(1e-40)
    assert np.isfinite(ge)
