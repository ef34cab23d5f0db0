"""Comparison rules shared by the GPU parity tests.

Tolerances:
  * attention outputs and compressed values (bf16 results of fp32 arithmetic on
    bf16/e4m3 inputs): max-abs error <= 2e-2 and relative L2 error <= 5e-3
    against the float64 oracle;
  * log-sum-exp: max-abs error <= 4e-3.  The tensor-core kernels sum the
    probabilities after rounding them to bf16 (the same values weight V), and a
    round to nearest moves a value by at most half an ulp, 2^-8 relative; so the
    sum is off by at most 2^-8 relative and ln of it by at most
    -ln(1 - 2^-8) = 3.92e-3 (fp32 accumulation and exp2 add ~1e-6);
  * E4M3 codes written by the compression epilogue: within one code step of the
    oracle's round-to-nearest-even code of its float64 value; scales rel 1e-5;
  * top-k index sets: identical, except rows where the oracle's k-th and
    (k+1)-th best scores differ by less than 1e-3 relative; there the GPU set
    must be a valid top-k of the oracle's scores within that band.
"""
from __future__ import annotations

import numpy as np
import torch

MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 4e-3
TIE_REL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def assert_close(got: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, rel_l2=REL_L2):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    ma = float(err.max()) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rl = float(np.linalg.norm(got - ref)) / den if den > 0 else float(np.linalg.norm(got - ref))
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max_abs={ma:.3e} rel_l2={rl:.3e}"
    return ma, rl


def assert_lse(got: np.ndarray, ref: np.ndarray, what: str):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    inf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), inf_ref), f"{what}: -inf pattern differs"
    if (~inf_ref).any():
        ma = float(np.abs(got[~inf_ref] - ref[~inf_ref]).max())
        assert ma <= LSE_ABS, f"{what}: lse max_abs={ma:.3e}"


def e4m3_ordinal(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def check_topk(got_idx: np.ndarray, scores: np.ndarray, ref_idx: np.ndarray, k: int, what: str) -> np.ndarray:
    """Checks GPU index lists against the oracle; returns a bool mask of rows with identical sets.

    got_idx, ref_idx: [..., k]; scores: oracle float64 scores [..., N] (-inf = not visible).
    A row may differ from the oracle's only where its k-th and (k+1)-th best
    scores lie within the tie band; there the GPU list must still be a top-k of
    the oracle's scores up to that band: k distinct visible entries in ascending
    order, none scoring below s_k - band, and every entry scoring above
    s_k + band among them.
    """
    got = np.asarray(got_idx).reshape(-1, k)
    ref = np.asarray(ref_idx).reshape(-1, k)
    sc = np.asarray(scores).reshape(got.shape[0], -1)
    same = np.all(got == ref, axis=1)
    for r in np.flatnonzero(~same):
        row = sc[r]
        vis = np.isfinite(row)
        nv = int(vis.sum())
        v = np.sort(row[vis])[::-1]
        assert nv > k, f"{what}: row {r} differs although every visible entry fits (nv={nv})"
        sk, sk1 = v[k - 1], v[k]
        band = TIE_REL * max(abs(sk), 1e-30)
        assert abs(sk - sk1) < band, (
            f"{what}: row {r} differs outside the tie band (s_k={sk}, s_k+1={sk1}); "
            f"extra={sorted(set(got[r]) - set(ref[r]))[:8]} missing={sorted(set(ref[r]) - set(got[r]))[:8]}")
        g = got[r]
        assert np.all(g >= 0) and np.all(g < row.shape[0]), f"{what}: row {r} has padding or out-of-range ids"
        assert np.all(np.diff(g) > 0), f"{what}: row {r} not ascending/unique"
        assert np.all(vis[g]), f"{what}: row {r} selects an invisible entry"
        assert row[g].min() >= sk - band, f"{what}: row {r} selects an entry below the band"
        must = np.flatnonzero(vis & (row > sk + band))
        missing = np.setdiff1d(must, g)
        assert missing.size == 0, f"{what}: row {r} drops entries above the band: {missing[:8].tolist()}"
    return same
