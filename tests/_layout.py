"""Test-only readers of the library's documented byte layouts (include/sharq.h).

These only move bytes around (no arithmetic of the method); they let a test
compare the GPU's tiled scale buffers with the oracle's row-major scales.
"""
import numpy as np


def untile_scales(buf, rows: int, s: int) -> np.ndarray:
    """Row-major (rows, s) view of a tiled scale buffer: blocks of 128 rows x 4
    scales, 512 bytes each, row-block major; inside a block, row r / scale j at
    (r % 32) * 16 + ((r // 32) % 4) * 4 + j."""
    b = np.asarray(buf, dtype=np.uint8)
    rb, sb = (rows + 127) // 128, (s + 3) // 4
    # byte offset inside a block = r0 * 16 + r1 * 4 + j  with r = 32 * r1 + r0
    blk = b[: rb * sb * 512].reshape(rb, sb, 32, 4, 4)   # [rowblk][sblk][r0][r1][j]
    out = blk.transpose(0, 3, 2, 1, 4).reshape(rb * 128, sb * 4)  # rows = rowblk*128 + r1*32 + r0
    return out[:rows, :s]


def tile_scales(a: np.ndarray) -> np.ndarray:
    """Inverse of untile_scales for arrays whose shape is already padded."""
    rows, s = a.shape
    rb, sb = rows // 128, s // 4
    blk = a.reshape(rb, 4, 32, sb, 4).transpose(0, 3, 2, 1, 4)
    return np.ascontiguousarray(blk).reshape(-1)
