"""Scale-factor storage order of the oracle (test infrastructure; see the package header).

The method fixes one UE4M3 scale per 16 values along K; where those bytes sit
in memory is fixed by the consumer, the block-scaled tensor-core MMA of the
target GPU, not by the pages.  The order used by the library (and stated in
its public header) is the one that MMA's scale-factor copy expects:

  * rows are grouped in blocks of 128 and scale columns (kk = k // 16) in
    blocks of 4, giving 512-byte tiles of 128 rows x 4 scales;
  * tiles are stored with the K-tile index fastest:
        tile = (row // 128) * (KS // 4) + kk // 4          (KS = K / 16)
  * inside a tile, row r and scale column kk sit at byte
        (r % 32) * 16 + ((r // 32) % 4) * 4 + (kk % 4)
  * rows past the last real row (up to the next multiple of 128) are padding
    and hold zero.

Pins: ``sf_offsets`` is a bijection onto [0, padded size) (tests); the
order itself is pinned on the GPU by the block-scaled GEMM: a wrong order
would pair codes with the wrong scales and fail the output parity tests.
"""
from __future__ import annotations

import numpy as np


def sf_padded_rows(rows: int) -> int:
    return -(-rows // 128) * 128


def sf_bytes(rows: int, K: int) -> int:
    """Size in bytes of the scale-factor buffer for a rows x K operand."""
    return sf_padded_rows(rows) * (K // 16)


def sf_offsets(rows: int, KS: int) -> np.ndarray:
    """Byte offset of scale (r, kk) for every r < rows, kk < KS (KS % 4 == 0)."""
    if KS % 4:
        raise ValueError("K must be a multiple of 64")
    r = np.arange(rows)[:, None]
    kk = np.arange(KS)[None, :]
    tile = (r // 128) * (KS // 4) + kk // 4
    return tile * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (kk % 4)


def sf_to_storage(scales: np.ndarray) -> np.ndarray:
    """rows x KS scale matrix -> flat uint8 buffer in the MMA's storage order (padding zero)."""
    scales = np.asarray(scales, dtype=np.uint8)
    rows, KS = scales.shape
    out = np.zeros(sf_padded_rows(rows) * KS, dtype=np.uint8)
    out[sf_offsets(rows, KS)] = scales
    return out


def sf_from_storage(buf: np.ndarray, rows: int, KS: int) -> np.ndarray:
    """Inverse of ``sf_to_storage`` for the first ``rows`` rows."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    return buf[sf_offsets(rows, KS)]
