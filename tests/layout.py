"""Host-side index helpers for the tests: unpack packed E2M1 codes and map
the MMA-tiled scale layout back to row-major.  Pure index arithmetic, stated
in include/nvfp4rac.h (nvfp4_tensor layout)."""
import numpy as np


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """uint8 [rows, cols/2] -> uint8 [rows, cols]; element 2j = low nibble."""
    p = np.asarray(packed, np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def tiled_scale_index(rows: int, cols: int) -> np.ndarray:
    """Byte offset of every (row, block) scale in the MMA-tiled layout."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    c = np.arange(cols // 16, dtype=np.int64)[None, :]
    k4 = -(-cols // 64)
    return ((r >> 7) * k4 + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3)


def untile_scales(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    return np.asarray(buf, np.uint8)[tiled_scale_index(rows, cols)]


def tiled_padding_mask(rows: int, cols: int) -> np.ndarray:
    """True for bytes of a tiled scale buffer that hold no (row, block)."""
    n = (-(-rows // 128)) * 128 * (-(-cols // 64)) * 4
    used = np.zeros(n, bool)
    used[tiled_scale_index(rows, cols).ravel()] = True
    return ~used
