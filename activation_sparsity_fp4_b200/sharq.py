"""Thin Python binding of ``include/sharq.h`` (ctypes).

Every function named ``sharq_*`` here calls the C function of the same name in
``_lib/libsharq.so``; the classes only allocate the caller-owned device
buffers (PyTorch tensors, the library allocates nothing) and marshal pointers,
shapes and the current CUDA stream.  All arithmetic runs in the CUDA kernels.
There is no CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build_ext

MXFP4, NVFP4 = 0, 1
NM_2_4, NM_4_8_PAIR, NM_8_16, NM_8_16_PAIR = 0, 1, 2, 3
F32, BF16 = 0, 1
FORMATS = {"mxfp4": MXFP4, "nvfp4": NVFP4}
PATTERNS = {"2:4": NM_2_4, "4:8pair": NM_4_8_PAIR, "8:16": NM_8_16, "8:16pair": NM_8_16_PAIR}
STATUS = {0: "SHARQ_OK", 1: "SHARQ_ERR_INVALID", 2: "SHARQ_ERR_UNSUPPORTED", 3: "SHARQ_ERR_CUDA",
          4: "SHARQ_ERR_TIMEOUT", 5: "SHARQ_ERR_WORKSPACE"}
SYMBOLS = ["sharq_weight_sizes", "sharq_prepared_sizes", "sharq_quantize_weight", "sharq_prepare", "sharq_linear",
           "sharq_linear_paths", "sharq_linear_grouped", "sharq_sync_status", "sharq_selftest_wait_timeout",
           "sharq_last_error", "sharq_launch_count", "sharq_prepare_noalloc", "sharq_prepare_swiglu",
           "sharq_gather_prepared", "sharq_linear_ws", "sharq_linear_workspace_size",
           "sharq_linear_grouped_gather"]
NOALLOC_MAX_ROWS = 65536  # SHARQ_NOALLOC_MAX_ROWS of the C header


class SharqError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class sharq_weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales_dense", ctypes.c_void_p), ("scales_sparse", ctypes.c_void_p),
                ("tensor", ctypes.c_void_p), ("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("experts", ctypes.c_int32), ("fmt", ctypes.c_int)]


class sharq_prepared(ctypes.Structure):
    _fields_ = [("meta", ctypes.c_void_p), ("bb_codes", ctypes.c_void_p), ("bb_scales", ctypes.c_void_p),
                ("res_codes", ctypes.c_void_p), ("res_scales", ctypes.c_void_p), ("tensor", ctypes.c_void_p),
                ("t", ctypes.c_int64), ("k", ctypes.c_int64), ("fmt", ctypes.c_int), ("pat", ctypes.c_int)]


_lib = None


def library_path() -> str:
    return build_ext.LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        path = build_ext.LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m activation_sparsity_fp4_b200.build_ext` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(path)
        P, I64, I32, I, F, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_float,
                                 ctypes.POINTER(ctypes.c_size_t))
        sig = {
            "sharq_weight_sizes": [I64, I64, I, SZ, SZ, SZ],
            "sharq_prepared_sizes": [I64, I64, I, I, SZ, SZ, SZ, SZ, SZ, SZ],
            "sharq_quantize_weight": [P, I, ctypes.POINTER(sharq_weight), P],
            "sharq_prepare": [P, I, P, F, F, ctypes.POINTER(sharq_prepared), P, ctypes.c_size_t, P],
            "sharq_prepare_noalloc": [P, I, P, F, F, ctypes.POINTER(sharq_prepared), P],
            "sharq_prepare_swiglu": [P, P, I, F, ctypes.POINTER(sharq_prepared), P],
            "sharq_gather_prepared": [ctypes.POINTER(sharq_prepared), P, ctypes.POINTER(sharq_prepared), P],
            "sharq_linear_ws": [ctypes.POINTER(sharq_prepared), ctypes.POINTER(sharq_weight), P, I, P,
                                ctypes.c_size_t, P],
            "sharq_linear_workspace_size": [ctypes.POINTER(ctypes.c_size_t)],
            "sharq_linear": [ctypes.POINTER(sharq_prepared), ctypes.POINTER(sharq_weight), P, I, P],
            "sharq_linear_paths": [ctypes.POINTER(sharq_prepared), ctypes.POINTER(sharq_weight), P, I, I32, P],
            "sharq_linear_grouped": [ctypes.POINTER(sharq_prepared), ctypes.POINTER(sharq_weight), P, P, I, P],
            "sharq_linear_grouped_gather": [ctypes.POINTER(sharq_prepared), P, I64, ctypes.POINTER(sharq_weight), P,
                                            P, I, P],
            "sharq_sync_status": [P],
            "sharq_selftest_wait_timeout": [ctypes.c_uint64, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.sharq_last_error.restype = ctypes.c_char_p
        L.sharq_last_error.argtypes = []
        L.sharq_launch_count.restype = ctypes.c_uint64
        L.sharq_launch_count.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise SharqError(status, where, lib().sharq_last_error().decode())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _fmt(f) -> int:
    return FORMATS[f] if isinstance(f, str) else int(f)


def _pat(p) -> int:
    return PATTERNS[p] if isinstance(p, str) else int(p)


def _dt(d) -> int:
    if isinstance(d, torch.dtype):
        if d == torch.bfloat16:
            return BF16
        if d == torch.float32:
            return F32
        raise ValueError(f"unsupported dtype {d}")
    return int(d)


# ------------------------------------------------------- same-name wrappers
def sharq_weight_sizes(n: int, k: int, fmt) -> tuple[int, int, int]:
    out = [ctypes.c_size_t() for _ in range(3)]
    _check(lib().sharq_weight_sizes(n, k, _fmt(fmt), *[ctypes.byref(o) for o in out]), "sharq_weight_sizes")
    return tuple(o.value for o in out)


def sharq_prepared_sizes(t: int, k: int, fmt, pat) -> tuple[int, int, int, int, int, int]:
    out = [ctypes.c_size_t() for _ in range(6)]
    _check(lib().sharq_prepared_sizes(t, k, _fmt(fmt), _pat(pat), *[ctypes.byref(o) for o in out]),
           "sharq_prepared_sizes")
    return tuple(o.value for o in out)


def sharq_quantize_weight(w_ptr: int, w_dt, out: sharq_weight, stream=None):
    _check(lib().sharq_quantize_weight(ctypes.c_void_p(w_ptr), _dt(w_dt), ctypes.byref(out), _stream(stream)),
           "sharq_quantize_weight")


def sharq_prepare(x_ptr: int, x_dt, gamma_ptr, eps: float, act_amax: float, out: sharq_prepared, workspace_ptr=None,
                  workspace_bytes: int = 0, stream=None):
    _check(lib().sharq_prepare(ctypes.c_void_p(x_ptr), _dt(x_dt), ctypes.c_void_p(gamma_ptr) if gamma_ptr else None,
                               float(eps), float(act_amax), ctypes.byref(out),
                               ctypes.c_void_p(workspace_ptr) if workspace_ptr else None, workspace_bytes,
                               _stream(stream)), "sharq_prepare")


def sharq_prepare_noalloc(x_ptr: int, x_dt, gamma_ptr, eps: float, act_amax: float, out: sharq_prepared,
                          stream=None):
    """sharq_prepare with the library's static per-row scratch: nothing is
    allocated, t <= NOALLOC_MAX_ROWS, first call per device before any stream
    capture, overlapping calls on one device race."""
    _check(lib().sharq_prepare_noalloc(ctypes.c_void_p(x_ptr), _dt(x_dt),
                                       ctypes.c_void_p(gamma_ptr) if gamma_ptr else None, float(eps), float(act_amax),
                                       ctypes.byref(out), _stream(stream)), "sharq_prepare_noalloc")


def sharq_prepare_swiglu(gate_ptr: int, up_ptr: int, dt, act_amax: float, out: sharq_prepared, stream=None):
    _check(lib().sharq_prepare_swiglu(ctypes.c_void_p(gate_ptr), ctypes.c_void_p(up_ptr), _dt(dt), float(act_amax),
                                      ctypes.byref(out), _stream(stream)), "sharq_prepare_swiglu")


def sharq_gather_prepared(src: sharq_prepared, rows_ptr: int, dst: sharq_prepared, stream=None):
    _check(lib().sharq_gather_prepared(ctypes.byref(src), ctypes.c_void_p(rows_ptr), ctypes.byref(dst),
                                       _stream(stream)), "sharq_gather_prepared")


def sharq_linear(a: sharq_prepared, w: sharq_weight, y_ptr: int, y_dt, stream=None):
    _check(lib().sharq_linear(ctypes.byref(a), ctypes.byref(w), ctypes.c_void_p(y_ptr), _dt(y_dt), _stream(stream)),
           "sharq_linear")


def sharq_linear_ws(a: sharq_prepared, w: sharq_weight, y_ptr: int, y_dt, ws_ptr: int, ws_bytes: int, stream=None):
    _check(lib().sharq_linear_ws(ctypes.byref(a), ctypes.byref(w), ctypes.c_void_p(y_ptr), _dt(y_dt),
                                 ctypes.c_void_p(ws_ptr), ctypes.c_size_t(ws_bytes), _stream(stream)),
           "sharq_linear_ws")


def sharq_linear_workspace_size() -> int:
    out = ctypes.c_size_t(0)
    _check(lib().sharq_linear_workspace_size(ctypes.byref(out)), "sharq_linear_workspace_size")
    return int(out.value)


def sharq_linear_paths(a: sharq_prepared, w: sharq_weight, y_ptr: int, y_dt, paths: int, stream=None):
    _check(lib().sharq_linear_paths(ctypes.byref(a), ctypes.byref(w), ctypes.c_void_p(y_ptr), _dt(y_dt), paths,
                                    _stream(stream)), "sharq_linear_paths")


def sharq_linear_grouped(a: sharq_prepared, w: sharq_weight, offsets_ptr: int, y_ptr: int, y_dt, stream=None):
    _check(lib().sharq_linear_grouped(ctypes.byref(a), ctypes.byref(w), ctypes.c_void_p(offsets_ptr),
                                      ctypes.c_void_p(y_ptr), _dt(y_dt), _stream(stream)), "sharq_linear_grouped")


def sharq_linear_grouped_gather(tokens: sharq_prepared, rows_ptr: int, routed_rows: int, w: sharq_weight,
                                offsets_ptr: int, y_ptr: int, y_dt, stream=None):
    _check(lib().sharq_linear_grouped_gather(ctypes.byref(tokens), ctypes.c_void_p(rows_ptr), int(routed_rows),
                                             ctypes.byref(w), ctypes.c_void_p(offsets_ptr), ctypes.c_void_p(y_ptr),
                                             _dt(y_dt), _stream(stream)), "sharq_linear_grouped_gather")


def sharq_sync_status(stream=None):
    _check(lib().sharq_sync_status(_stream(stream)), "sharq_sync_status")


def sharq_selftest_wait_timeout(timeout_ns: int, stream=None):
    _check(lib().sharq_selftest_wait_timeout(int(timeout_ns), _stream(stream)), "sharq_selftest_wait_timeout")


def sharq_last_error() -> str:
    return lib().sharq_last_error().decode()


def sharq_launch_count(reset: bool = False) -> int:
    return int(lib().sharq_launch_count(1 if reset else 0))


# ------------------------------------------------------------ buffer owners
def _alloc(nbytes: int, device) -> torch.Tensor:
    # 256-byte aligned (PyTorch's caching allocator aligns blocks to 512 bytes)
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


class FP4Weight:
    """Device buffers of a shared FP4 weight (one or ``experts`` stacked)."""

    def __init__(self, n: int, k: int, fmt, experts: int = 1, device="cuda"):
        self.n, self.k, self.fmt, self.experts = n, k, _fmt(fmt), experts
        c, d, s = sharq_weight_sizes(n, k, self.fmt)
        self.codes = _alloc(c * experts, device)
        self.scales_dense = _alloc(d * experts, device)
        self.scales_sparse = _alloc(s * experts, device)
        self.tensor = torch.zeros(3 * experts, dtype=torch.float32, device=device)
        self.struct = sharq_weight(self.codes.data_ptr(), self.scales_dense.data_ptr(),
                                   self.scales_sparse.data_ptr(), self.tensor.data_ptr(), n, k, experts, self.fmt)

    @classmethod
    def quantize(cls, w: torch.Tensor, fmt, stream=None) -> "FP4Weight":
        """w: (n, k) or (experts, n, k), bf16 or fp32, on the GPU."""
        w = w.contiguous()
        experts = w.shape[0] if w.dim() == 3 else 1
        n, k = w.shape[-2], w.shape[-1]
        obj = cls(n, k, fmt, experts, w.device)
        sharq_quantize_weight(w.data_ptr(), w.dtype, obj.struct, stream)
        obj._src = w  # keep the source alive until the stream has consumed it
        return obj


class Prepared:
    """Device buffers of prepared activations for t rows."""

    def __init__(self, t: int, k: int, fmt, pat, device="cuda"):
        self.t, self.k, self.fmt, self.pat = t, k, _fmt(fmt), _pat(pat)
        m, bc, bs, rc, rs, ws = sharq_prepared_sizes(t, k, self.fmt, self.pat)
        self.meta = _alloc(m, device)
        self.bb_codes = _alloc(bc, device)
        self.bb_scales = _alloc(bs, device)
        self.res_codes = _alloc(rc, device)
        self.res_scales = _alloc(rs, device)
        self.tensor = torch.zeros(3, dtype=torch.float32, device=device)
        self.workspace = _alloc(ws, device) if ws else None
        self.struct = sharq_prepared(self.meta.data_ptr(), self.bb_codes.data_ptr(), self.bb_scales.data_ptr(),
                                     self.res_codes.data_ptr(), self.res_scales.data_ptr(), self.tensor.data_ptr(),
                                     t, k, self.fmt, self.pat)


def prepare(x: torch.Tensor, fmt, pat, gamma: torch.Tensor | None = None, eps: float = 1e-6, act_amax: float = 0.0,
            out: Prepared | None = None, stream=None, use_workspace: bool = True) -> Prepared:
    """Fused preprocessing of x (t, k) on the GPU; returns (or fills) a Prepared.
    use_workspace=False runs without the per-row scratch (same results)."""
    x = x.contiguous()
    t, k = x.shape
    if out is None:
        out = Prepared(t, k, fmt, pat, x.device)
    if gamma is not None:
        gamma = gamma.to(x.dtype).contiguous()
    ws = out.workspace if use_workspace else None
    sharq_prepare(x.data_ptr(), x.dtype, gamma.data_ptr() if gamma is not None else None, eps, act_amax, out.struct,
                  ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, stream)
    return out


def prepare_swiglu(gate: torch.Tensor, up: torch.Tensor, fmt, pat, act_amax: float = 0.0,
                   out: Prepared | None = None, stream=None) -> Prepared:
    """Preprocessing of h = SiLU(gate) * up (t, k), formed inside the kernel."""
    gate, up = gate.contiguous(), up.to(gate.dtype).contiguous()
    assert gate.shape == up.shape
    t, k = gate.shape
    if out is None:
        out = Prepared(t, k, fmt, pat, gate.device)
    sharq_prepare_swiglu(gate.data_ptr(), up.data_ptr(), gate.dtype, act_amax, out.struct, stream)
    return out


def gather_prepared(src: Prepared, rows: torch.Tensor, out: Prepared | None = None, stream=None) -> Prepared:
    """Prepared rows laid out again: row i of the result is src row rows[i] (a zero row for
    rows[i] < 0)."""
    rows = rows.to(torch.int32).contiguous()
    if out is None:
        out = Prepared(rows.numel(), src.k, src.fmt, src.pat, src.meta.device)
    sharq_gather_prepared(src.struct, rows.data_ptr(), out.struct, stream)
    return out


def linear_workspace(device="cuda") -> torch.Tensor:
    """A zero-filled stream-K workspace for `linear(..., workspace=...)` on this device."""
    with torch.cuda.device(torch.device(device)):
        return torch.zeros(sharq_linear_workspace_size(), dtype=torch.uint8, device=device)


def linear(a: Prepared, w: FP4Weight, out_dtype=torch.bfloat16, out: torch.Tensor | None = None, paths: int = 3,
           stream=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y = the sparse backbone GEMM plus the dense residual GEMM, (t, n).  With a
    workspace (see `linear_workspace`) the CTA-pair GEMM may split its K loops
    over every SM pair (stream-K)."""
    if out is None:
        out = torch.empty((a.t, w.n), dtype=out_dtype, device=a.meta.device)
    if workspace is not None:
        assert paths == 3, "the stream-K form runs both paths"
        sharq_linear_ws(a.struct, w.struct, out.data_ptr(), out.dtype, workspace.data_ptr(),
                        workspace.numel() * workspace.element_size(), stream)
    elif paths == 3:
        sharq_linear(a.struct, w.struct, out.data_ptr(), out.dtype, stream)
    else:
        sharq_linear_paths(a.struct, w.struct, out.data_ptr(), out.dtype, paths, stream)
    return out


def linear_grouped(a: Prepared, w: FP4Weight, offsets: torch.Tensor, out_dtype=torch.bfloat16,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.zeros((a.t, w.n), dtype=out_dtype, device=a.meta.device)
    offsets = offsets.to(torch.int32).contiguous()
    sharq_linear_grouped(a.struct, w.struct, offsets.data_ptr(), out.data_ptr(), out.dtype, stream)
    return out


def linear_grouped_gather(tokens: Prepared, rows: torch.Tensor, w: FP4Weight, offsets: torch.Tensor,
                          out_dtype=torch.bfloat16, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Grouped linear over routed rows read by index from the token-prepared buffers
    (rows[r] = token of routed row r, < 0 for a padding row)."""
    rows = rows.to(torch.int32).contiguous()
    if out is None:
        out = torch.zeros((rows.numel(), w.n), dtype=out_dtype, device=tokens.meta.device)
    offsets = offsets.to(torch.int32).contiguous()
    sharq_linear_grouped_gather(tokens.struct, rows.data_ptr(), rows.numel(), w.struct, offsets.data_ptr(),
                                out.data_ptr(), out.dtype, stream)
    return out
