"""Test helpers: torch <-> numpy marshalling for the CUDA path and reading
its blocked MXFP8 scale layout back into plain [rows, K/32] order, plus the
comparison metrics written in the tests' tolerances.  Shares nothing with
the oracle."""
from __future__ import annotations

import numpy as np


def sf_unblock(sf: np.ndarray, groups: int, rows: int, K: int) -> np.ndarray:
    """Blocked scale bytes (layout documented in include/moe_mxfp8.h) ->
    uint8 [groups, rows, K/32]."""
    RT, KT, nkb = -(-rows // 128), -(-K // 128), K // 32
    g = np.arange(groups)[:, None, None]
    r = np.arange(rows)[None, :, None]
    kb = np.arange(nkb)[None, None, :]
    off = ((g * RT + r // 128) * KT + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4
    return np.asarray(sf)[off]


def sf_padding_offsets(groups: int, rows: int, K: int) -> np.ndarray:
    """Offsets of the blocked layout that belong to no (row, block)."""
    RT, KT, nkb = -(-rows // 128), -(-K // 128), K // 32
    total = groups * RT * KT * 512
    used = np.zeros(total, bool)
    g = np.arange(groups)[:, None, None]
    r = np.arange(rows)[None, :, None]
    kb = np.arange(nkb)[None, None, :]
    off = ((g * RT + r // 128) * KT + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4
    used[off.reshape(-1)] = True
    return np.flatnonzero(~used)


def e4m3_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance between E4M3 codes in steps of the ordered code line
    (+0 and -0 coincide)."""
    def line(c):
        c = c.astype(np.int64)
        m = c & 0x7F
        return np.where(c & 0x80, -m, m)
    return np.abs(line(a) - line(b))


def rel_max_over_rms(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max |gpu - ref| / rms(ref)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.abs(gpu - ref)) / rms) if ref.size else 0.0


def bf16_to_f64(t) -> np.ndarray:
    """torch bf16 tensor (any device) -> float64 numpy."""
    return t.float().cpu().numpy().astype(np.float64)


def requant_mismatch(gpu_codes, gpu_sf, ref_codes, ref_sf, ref_amax):
    """Compare requantised MXFP8 rows against the oracle.

    Returns (fraction of differing elements, max ulp distance among elements
    of blocks whose scales agree, number of blocks whose scales differ
    without the oracle's amax lying within 1e-5 relative of a scale
    boundary).  Every element of a block with a differing scale counts as
    differing."""
    n, K = ref_codes.shape
    nb = K // 32
    sf_diff = gpu_sf != ref_sf                                   # [n, nb]
    # scale boundaries: amax = 448 * 2^s exactly
    with np.errstate(divide="ignore"):
        ratio = ref_amax / 448.0
        near = np.zeros_like(ratio, dtype=bool)
        pos = ratio > 0
        lg = np.log2(ratio[pos])
        near[pos] = np.abs(2.0 ** np.round(lg) / ratio[pos] - 1.0) <= 1e-5
    bad_scale_blocks = int(np.sum(sf_diff & ~near))
    d = e4m3_ulp_distance(gpu_codes, ref_codes).reshape(n, nb, 32)
    same = ~sf_diff
    elem_diff = (d > 0) & same[:, :, None]
    n_diff = int(np.sum(elem_diff)) + int(np.sum(sf_diff)) * 32
    max_ulp = int(d[same].max()) if np.any(same) else 0
    return n_diff / float(n * K), max_ulp, bad_scale_blocks
