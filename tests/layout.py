"""Index map of the E8M0 scale "MMA tile layout" documented in include/macaq.h, written
from that documentation (no library code), used to compare the CUDA path's scales with
the oracle's row-major [rows][K/32] scales."""
import numpy as np


def padded_blocks(K: int) -> int:
    return 8 * ((K + 255) // 256)


def scale_bytes(rows: int, K: int) -> int:
    return ((rows + 127) // 128) * 128 * padded_blocks(K)


def scale_index(rows: int, K: int, nblocks: int | None = None) -> np.ndarray:
    """int64 [rows][nblocks] offsets of (row r, block kb); nblocks defaults to K/32."""
    kbp = padded_blocks(K)
    nb = K // 32 if nblocks is None else nblocks
    r = np.arange(rows, dtype=np.int64)[:, None]
    kb = np.arange(nb, dtype=np.int64)[None, :]
    return ((r // 128) * (kbp // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4


def tiled_to_rowmajor(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return np.asarray(buf)[scale_index(rows, K)]


def rowmajor_to_tiled(S: np.ndarray, rows: int, K: int) -> np.ndarray:
    out = np.zeros(scale_bytes(rows, K), np.uint8)
    out[scale_index(rows, K)] = S
    return out


def padded_block_bytes(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Bytes of the padded blocks (kb >= K/32) of real rows; writers must zero them."""
    kbp = padded_blocks(K)
    idx = scale_index(rows, K, kbp)[:, K // 32:]
    return np.asarray(buf)[idx]


def rows_of_tiled(buf: np.ndarray, rows, K: int) -> np.ndarray:
    """A scale buffer in the same layout holding only the listed rows (in that order), padded
    blocks included, so a sample of rows can be compared like a whole matrix."""
    kbp = padded_blocks(K)
    r = np.asarray(rows, dtype=np.int64)[:, None]
    kb = np.arange(kbp, dtype=np.int64)[None, :]
    src = ((r // 128) * (kbp // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    out = np.zeros(scale_bytes(len(rows), K), np.uint8)
    out[scale_index(len(rows), K, kbp)] = np.asarray(buf)[src]
    return out
