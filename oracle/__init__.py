"""CPU oracle for the SharQ sparse-dense FP4 linear layer.

TEST INFRASTRUCTURE ONLY: tests/, the smoke check in ``__graft_entry__`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package; the product path (``activation_sparsity_fp4_b200``) never does, and
this package never imports the product.  Shared with the product: only the
seeded input generators in ``activation_sparsity_fp4_b200.workloads``.

The arithmetic lives in ``sharq_oracle.c`` (plain C, fp32 round-to-nearest
steps, compiled with ``-ffp-contract=off``).  This module compiles it with gcc
on first use, marshals numpy arrays, and adds the fp64 reference GEMM
(``linear_ref``: a numpy fp64 matmul over the exactly decoded operands).

Sources (SharQ, arXiv 2606.26587, abstract / Section 1 / Section 2.2;
"From 2:4 to 8:16 sparsity patterns..." abstract; Huawei problem 137-2):
see the header of ``sharq_oracle.c`` for which step follows which passage.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sharq_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

MXFP4, NVFP4 = 0, 1
NM_2_4, NM_4_8_PAIR, NM_8_16, NM_8_16_PAIR = 0, 1, 2, 3
FORMATS = {"mxfp4": MXFP4, "nvfp4": NVFP4}
# "8:16pair": the 8:16 selection re-packed into the 4:8 pair layout
PATTERNS = {"2:4": NM_2_4, "4:8pair": NM_4_8_PAIR, "8:16": NM_8_16, "8:16pair": NM_8_16_PAIR}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so`` (gcc, -O2, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        sig = {
            "orc_e2m1_encode_n": (None, [P, I64, P]),
            "orc_e4m3_encode_n": (None, [P, I64, P]),
            "orc_floor_log2_n": (None, [P, I64, P]),
            "orc_e2m1_decode": (F, [ctypes.c_uint8]),
            "orc_e4m3_decode": (F, [ctypes.c_uint8]),
            "orc_e8m0_decode": (F, [ctypes.c_uint8]),
            "orc_rms_rstd": (F, [P, I64, F]),
            "orc_mask_rows": (None, [P, I64, I64, I, P]),
            "orc_rows_amax": (F, [P, I64, I64, P, F]),
            "orc_tensor_scale": (None, [F, P, P]),
            "orc_quant_block": (ctypes.c_uint8, [P, I, I, F, P]),
            "orc_quant_blocks_n": (None, [P, I64, I, I, F, P, P]),
            "orc_prepare": (I, [P, I64, I64, P, F, I, I, F, P, P, P, P, P, P, P, P, P]),
            "orc_quantize_weight": (I, [P, I64, I64, I, P, P, P]),
            "orc_decode_prepared": (None, [P, P, P, P, P, I64, I64, I, I, P, P]),
            "orc_decode_weight": (None, [P, P, I64, I64, I, P]),
            "orc_meta_bytes_per_row": (I64, [I64, I]),
            "orc_exp": (F, [F]),
            "orc_silu": (F, [F]),
            "orc_swiglu": (None, [P, P, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def _pat(pat) -> int:
    return PATTERNS[pat] if isinstance(pat, str) else int(pat)


def block_size(fmt) -> int:
    """Elements per scale of a dense FP4 block: 32 (MXFP4) or 16 (NVFP4)."""
    return 32 if _fmt(fmt) == MXFP4 else 16


# ----------------------------------------------------------------- formats
def e2m1_encode(v) -> np.ndarray:
    v = _f32(v).ravel()
    out = np.empty(v.size, np.uint8)
    _load().orc_e2m1_encode_n(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_decode(codes) -> np.ndarray:
    lib = _load()
    return np.array([lib.orc_e2m1_decode(int(c)) for c in np.asarray(codes).ravel()], np.float32)


def e4m3_encode(v) -> np.ndarray:
    v = _f32(v).ravel()
    out = np.empty(v.size, np.uint8)
    _load().orc_e4m3_encode_n(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    return np.array([lib.orc_e4m3_decode(int(c)) for c in np.asarray(codes).ravel()], np.float32)


def e8m0_decode(codes) -> np.ndarray:
    lib = _load()
    return np.array([lib.orc_e8m0_decode(int(c)) for c in np.asarray(codes).ravel()], np.float32)


def floor_log2(v) -> np.ndarray:
    v = _f32(v).ravel()
    out = np.empty(v.size, np.int32)
    _load().orc_floor_log2_n(_ptr(v), v.size, _ptr(out))
    return out


# ------------------------------------------------------------------- steps
def rms_rstd(x_row, eps: float = 1e-6) -> float:
    x = _f32(x_row).ravel()
    return float(_load().orc_rms_rstd(_ptr(x), x.size, eps))


def mask(h, pat) -> np.ndarray:
    """Keep flags (uint8 0/1) of the N:M mask for each row of ``h`` (t x k)."""
    h = _f32(h)
    h2 = h.reshape(-1, h.shape[-1])
    keep = np.empty(h2.shape, np.uint8)
    _load().orc_mask_rows(_ptr(h2), h2.shape[0], h2.shape[1], _pat(pat), _ptr(keep))
    return keep.reshape(h.shape)


def tensor_scale(amax: float):
    ge, gd = ctypes.c_float(), ctypes.c_float()
    _load().orc_tensor_scale(amax, ctypes.byref(ge), ctypes.byref(gd))
    return ge.value, gd.value


def quant_block(v, fmt, g_enc: float = 1.0):
    """(scale_code, codes) of one block of values sharing a scale."""
    v = _f32(v).ravel()
    codes = np.empty(v.size, np.uint8)
    sc = _load().orc_quant_block(_ptr(v), v.size, _fmt(fmt), g_enc, _ptr(codes))
    return int(sc), codes


def quant_blocks(v, block: int, fmt, g_enc: float = 1.0):
    """Consecutive blocks of ``block`` values along the last axis, each with its own
    scale: (scale codes [..., n / block], E2M1 codes [..., n])."""
    v = _f32(v)
    flat = v.reshape(-1)
    assert flat.size % block == 0
    codes = np.empty(flat.size, np.uint8)
    scales = np.empty(flat.size // block, np.uint8)
    _load().orc_quant_blocks_n(_ptr(flat), flat.size // block, block, _fmt(fmt), g_enc, _ptr(codes), _ptr(scales))
    return scales.reshape(v.shape[:-1] + (v.shape[-1] // block,)), codes.reshape(v.shape)


def dequant_blocks(scales, codes, fmt, g_dec: float = 1.0) -> np.ndarray:
    """fp64 values of quant_blocks' output: E2M1 * block scale (exact) * g_dec."""
    lib = _load()
    e2 = np.array([lib.orc_e2m1_decode(c) for c in range(16)], np.float64)
    dec = lib.orc_e8m0_decode if _fmt(fmt) == MXFP4 else lib.orc_e4m3_decode
    sv = np.array([dec(c) for c in range(256)], np.float64)
    block = codes.shape[-1] // scales.shape[-1]
    return e2[codes] * np.repeat(sv[scales], block, axis=-1) * (1.0 if _fmt(fmt) == MXFP4 else float(g_dec))


def meta_bytes_per_row(k: int, pat) -> int:
    return int(_load().orc_meta_bytes_per_row(k, _pat(pat)))


def rows_amax(x, gamma=None, eps: float = 1e-6) -> float:
    x = _f32(x)
    g = None if gamma is None else _f32(gamma)
    return float(_load().orc_rows_amax(_ptr(x), x.shape[0], x.shape[1], _ptr(g), eps))


def exp(x) -> np.ndarray:
    """The oracle's fp32 exponential (Cody-Waite reduction + degree-7 Taylor), elementwise."""
    lib = _load()
    x = _f32(x)
    return np.array([lib.orc_exp(float(v)) for v in x.ravel()], np.float32).reshape(x.shape)


def swiglu(gate, up) -> np.ndarray:
    """h = SiLU(gate) * up in the oracle's fixed fp32 steps (inputs converted exactly to fp32)."""
    a, b = _f32(gate), _f32(up)
    assert a.shape == b.shape
    h = np.empty_like(a)
    _load().orc_swiglu(_ptr(a), _ptr(b), a.size, _ptr(h))
    return h


def prepare_swiglu(gate, up, fmt, pat, act_amax: float = 0.0, *, threads: int = 1, want_float: bool = False) -> dict:
    """Preprocessing of a down projection's input formed on the fly: h = SiLU(gate) * up
    (no RMSNorm), then the mask, backbone and residual of ``prepare``."""
    return prepare(swiglu(gate, up), fmt, pat, None, 1e-6, act_amax, threads=threads, want_float=want_float)


def prepare(x, fmt, pat, gamma=None, eps: float = 1e-6, act_amax: float = 0.0, *, threads: int = 1,
            want_float: bool = False) -> dict:
    """Whole preprocessing of ``x`` (t x k, converted exactly to fp32).

    Returns canonical outputs: ``meta``, ``bb_codes``, ``bb_scales``, ``res_codes``,
    ``res_scales`` (uint8, row-major, codes packed low nibble first) and ``tensor``
    = [amax, g_enc, g_dec].  With ``want_float`` also ``h``, ``bdeq``, ``rdeq`` (fp32).
    ``threads`` > 1 splits rows across threads after computing the NVFP4 tensor
    amax once, which gives bit-identical results (rows are independent given it).
    """
    lib = _load()
    f, p = _fmt(fmt), _pat(pat)
    x = _f32(x)
    t, k = x.shape
    g = None if gamma is None else _f32(gamma)
    b = block_size(f)
    mb = meta_bytes_per_row(k, p)
    out = {
        "meta": np.zeros((t, mb), np.uint8),
        "bb_codes": np.zeros((t, k // 2 if p == NM_8_16 else k // 4), np.uint8),
        "bb_scales": np.zeros((t, k // (2 * b)), np.uint8),
        "res_codes": np.zeros((t, k // 2), np.uint8),
        "res_scales": np.zeros((t, k // b), np.uint8),
        "tensor": np.zeros(3, np.float32),
    }
    fl = {}
    if want_float:
        fl = {n: np.zeros((t, k), np.float32) for n in ("h", "bdeq", "rdeq")}
    if f == NVFP4 and not act_amax > 0 and threads > 1 and t > 1:
        act_amax = rows_amax(x, g, eps)

    def run(r0: int, r1: int):
        tens = np.zeros(3, np.float32)
        sl = slice(r0, r1)
        args = [_ptr(x[sl]), r1 - r0, k, _ptr(g), eps, f, p, float(act_amax)]
        args += [_ptr(out[n][sl]) for n in ("meta", "bb_codes", "bb_scales", "res_codes", "res_scales")]
        args += [_ptr(tens)]
        args += [_ptr(fl[n][sl]) if want_float else None for n in ("h", "bdeq", "rdeq")]
        rc = lib.orc_prepare(*args)
        if rc != 0:
            raise ValueError(f"oracle prepare rejected t={t} k={k} fmt={fmt} pat={pat}")
        return tens

    if threads <= 1 or t <= 1:
        out["tensor"][:] = run(0, t)
    else:
        bounds = np.linspace(0, t, threads + 1).astype(int)
        with ThreadPoolExecutor(threads) as ex:
            tens = list(ex.map(lambda i: run(bounds[i], bounds[i + 1]),
                               [i for i in range(threads) if bounds[i] < bounds[i + 1]]))
        out["tensor"][:] = tens[0]
    out.update(fl)
    out["fmt"], out["pat"], out["t"], out["k"] = f, p, t, k
    return out


def quantize_weight(w, fmt) -> dict:
    """Shared FP4 weight: codes (n x k/2), scales per 2b logical K (n x k/(2b)), tensor."""
    lib = _load()
    f = _fmt(fmt)
    w = _f32(w)
    n, k = w.shape
    b = block_size(f)
    out = {
        "codes": np.zeros((n, k // 2), np.uint8),
        "scales": np.zeros((n, k // (2 * b)), np.uint8),
        "tensor": np.zeros(3, np.float32),
    }
    rc = lib.orc_quantize_weight(_ptr(w), n, k, f, _ptr(out["codes"]), _ptr(out["scales"]), _ptr(out["tensor"]))
    if rc != 0:
        raise ValueError(f"oracle quantize_weight rejected n={n} k={k}")
    out["fmt"], out["n"], out["k"] = f, n, k
    return out


def decode_prepared(prep: dict, rows=None):
    """Exact fp64 (backbone, residual) operands without tensor scales, t x k each."""
    lib = _load()
    t, k, f, p = prep["t"], prep["k"], prep["fmt"], prep["pat"]
    sel = np.arange(t) if rows is None else np.asarray(rows)
    parts = {n: np.ascontiguousarray(prep[n][sel]) for n in ("meta", "bb_codes", "bb_scales", "res_codes",
                                                               "res_scales")}
    bu = np.zeros((sel.size, k), np.float64)
    ru = np.zeros((sel.size, k), np.float64)
    lib.orc_decode_prepared(_ptr(parts["meta"]), _ptr(parts["bb_codes"]), _ptr(parts["bb_scales"]),
                            _ptr(parts["res_codes"]), _ptr(parts["res_scales"]), sel.size, k, f, p,
                            _ptr(bu), _ptr(ru))
    return bu, ru


def decode_weight(wq: dict) -> np.ndarray:
    lib = _load()
    wu = np.zeros((wq["n"], wq["k"]), np.float64)
    lib.orc_decode_weight(_ptr(np.ascontiguousarray(wq["codes"])), _ptr(np.ascontiguousarray(wq["scales"])),
                          wq["n"], wq["k"], wq["fmt"], _ptr(wu))
    return wu


def linear_ref(prep: dict, wq: dict, rows=None, wu: np.ndarray | None = None) -> np.ndarray:
    """fp64 reference of the layer output on the dequantized operands:
    Y = g_dec_x * g_dec_w * (B + R) . W^T, the sparse backbone product plus the
    dense residual product accumulated into it (SharQ abstract, Section 1)."""
    bu, ru = decode_prepared(prep, rows)
    if wu is None:
        wu = decode_weight(wq)
    alpha = float(prep["tensor"][2]) * float(wq["tensor"][2])
    return alpha * ((bu + ru) @ wu.T)
