"""CPU checks of the C-ABI boundary: the library loads, exports every entry
point that include/sharq.h declares, and rejects bad arguments on the host
(before any launch, so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from activation_sparsity_fp4_b200 import build_ext, sharq

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sharq.h")


@pytest.fixture(scope="module")
def L():
    build_ext.build()
    return sharq.lib()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:sharq_status|const char\*|uint64_t)\s+(sharq_\w+)\s*\(", text, re.M)))


def test_header_declares_the_entry_points():
    names = _declared()
    for required in ("sharq_quantize_weight", "sharq_prepare", "sharq_linear"):
        assert required in names
    assert set(names) == set(sharq.SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_weight_sizes(L):
    c, d, s = sharq.sharq_weight_sizes(4096, 4096, "nvfp4")
    assert c == 4096 * 4096 // 2
    assert d == 4096 * 4096 // 16  # one E4M3 per 16, no padding at this shape
    assert s == 4096 * 4096 // 32
    c, d, s = sharq.sharq_weight_sizes(4096, 14336, "mxfp4")
    assert (c, d, s) == (4096 * 14336 // 2, 4096 * 14336 // 32, 4096 * 14336 // 64)


def test_prepared_sizes_pad_rows_to_128(L):
    m, bc, bs, rc, rs, ws = sharq.sharq_prepared_sizes(16, 256, "mxfp4", "2:4")
    assert (m, bc, rc) == (128 * 256 // 8, 128 * 256 // 4, 128 * 256 // 2)
    assert bs == 512 and rs == 128 * 8 // 4 * 4  # 256/64 = 4 scales; 256/32 = 8 scales per row
    assert ws == 128 * 4  # one float per padded row
    m, bc, bs, rc, rs, ws = sharq.sharq_prepared_sizes(2048, 4096, "nvfp4", "4:8pair")
    assert m == 2048 * 4096 // 16 and bc == 2048 * 4096 // 4
    assert bs == 2048 * 4096 // 32 and rs == 2048 * 4096 // 16
    m, bc, bs, rc, rs, ws = sharq.sharq_prepared_sizes(100, 5120, "nvfp4", "8:16")
    assert bc == 128 * 5120 // 2 and bs == 128 * 5120 // 16 and m == 128 * 5120 // 8


@pytest.mark.parametrize("k,n", [(255, 256), (384, 256), (256, 128), (0, 256)])
def test_bad_shapes_are_rejected(L, k, n):
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_weight_sizes(n, k, "nvfp4")
    assert ei.value.status in (1, 2)


def test_bad_enums_and_pointers_are_rejected_without_launch(L):
    before = sharq.sharq_launch_count()
    with pytest.raises(sharq.SharqError):
        sharq.sharq_prepared_sizes(16, 256, 7, 0)
    w = sharq.sharq_weight(None, None, None, None, 256, 256, 1, 0)
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_quantize_weight(0, sharq.F32, w, 0)
    assert ei.value.status == 1
    a = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 16, 256, 1, 0)  # NVFP4 with 2:4
    wq = sharq.sharq_weight(16, 16, 16, 16, 256, 256, 1, 1)
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_linear(a, wq, 16, sharq.F32, 0)
    assert ei.value.status == 2
    a2 = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 16, 512, 1, 1)
    with pytest.raises(sharq.SharqError) as ei:  # k mismatch
        sharq.sharq_linear(a2, wq, 16, sharq.F32, 0)
    assert ei.value.status == 1
    a3 = sharq.sharq_prepared(8, 16, 16, 16, 16, 16, 16, 256, 1, 1)  # misaligned meta pointer
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_linear(a3, wq, 16, sharq.F32, 0)
    assert "aligned" in str(ei.value)
    assert sharq.sharq_launch_count() == before
    assert sharq.sharq_last_error() != ""


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(build_ext, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(sharq, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        sharq.lib()


def test_noalloc_limit_matches_header_and_rejects_on_host(L):
    text = open(HEADER).read()
    m = re.search(r"#define\s+SHARQ_NOALLOC_MAX_ROWS\s+(\d+)", text)
    assert m and int(m.group(1)) == sharq.NOALLOC_MAX_ROWS
    before = sharq.sharq_launch_count()
    a = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, sharq.NOALLOC_MAX_ROWS + 1, 256, 1, 1)
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_prepare_noalloc(16, sharq.BF16, None, 1e-6, 0.0, a, 0)
    assert ei.value.status == 5 and "static scratch" in str(ei.value)
    assert sharq.sharq_launch_count() == before


def test_gather_prepared_rejects_mismatch_on_host(L):
    """Source and destination must agree on k, format and pattern; checked before any launch."""
    before = sharq.sharq_launch_count()
    src = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 256, 512, 1, 1)
    for dst in (sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 128, 256, 1, 1),
                sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 128, 512, 0, 1),
                sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 128, 512, 1, 2)):
        with pytest.raises(sharq.SharqError) as ei:
            sharq.sharq_gather_prepared(src, 16, dst, 0)
        assert ei.value.status == 1
    with pytest.raises(sharq.SharqError):  # no index array
        sharq.sharq_gather_prepared(src, 0, sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 128, 512, 1, 1), 0)
    assert sharq.sharq_launch_count() == before


def test_linear_ws_requires_a_workspace(L):
    before = sharq.sharq_launch_count()
    a = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 256, 256, 1, 1)
    w = sharq.sharq_weight(16, 16, 16, 16, 256, 256, 1, 1)
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_linear_ws(a, w, 16, sharq.BF16, 0, 0, 0)
    assert ei.value.status == 5 and "workspace" in str(ei.value)
    assert sharq.sharq_launch_count() == before


def test_grouped_gather_rejects_on_host(L):
    """The in-GEMM row gather takes NVFP4 with the 4:8 pair only, routed rows in
    multiples of 128 and an index array; all checked before any launch."""
    before = sharq.sharq_launch_count()
    w = sharq.sharq_weight(16, 16, 16, 16, 256, 512, 4, 1)
    ok = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 300, 512, 1, 1)
    for tok, rows, routed, status in ((sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 300, 512, 0, 1), 16, 256, 2),
                                      (sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 300, 512, 1, 2), 16, 256, 2),
                                      (ok, 16, 200, 1), (ok, 0, 256, 1), (ok, 18, 256, 1)):
        with pytest.raises(sharq.SharqError) as ei:
            sharq.sharq_linear_grouped_gather(tok, rows, routed, w, 16, 16, sharq.BF16, 0)
        assert ei.value.status == status, str(ei.value)
    assert sharq.sharq_launch_count() == before


def test_empty_inputs_are_rejected_without_launch(L):
    """Zero rows (and a non-positive row count in the size queries) is an argument
    error on the host: prepare, linear, the grouped and gathered forms and the
    row gather all refuse it before any launch."""
    before = sharq.sharq_launch_count()
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_prepared_sizes(0, 256, "nvfp4", "4:8pair")
    assert ei.value.status == 1
    empty = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 0, 256, 1, 1)
    wq = sharq.sharq_weight(16, 16, 16, 16, 256, 256, 1, 1)
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_prepare(16, sharq.BF16, None, 1e-6, 0.0, empty, None, 0, 0)
    assert ei.value.status == 1
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_linear(empty, wq, 16, sharq.BF16, 0)
    assert ei.value.status == 1
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_linear_grouped(empty, wq, 16, 16, sharq.BF16, 0)
    assert ei.value.status == 1
    ok = sharq.sharq_prepared(16, 16, 16, 16, 16, 16, 128, 256, 1, 1)
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_gather_prepared(ok, 16, empty, 0)
    assert ei.value.status == 1
    assert sharq.sharq_launch_count() == before
