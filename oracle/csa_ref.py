"""CPU oracle for Compressed Sparse Attention (CSA) and Heavily Compressed Attention (HCA).

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain, float64 statement of
what the CUDA library computes.  Only the test suite, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline leg may import it; the library never does, and
this module imports nothing from the library (it shares only the seeded input
generator, which holds none of the method's arithmetic).

Source of the method: the DeepSeek-V4 paper summary on hyper.ai
(papers/2606.19348), section "方法" (Method):
  * CSA paragraph -- every m tokens of the KV cache are compressed into one
    entry with learnable compression weights and a position bias; a "lightning
    indexer" picks the top-k compressed entries for the core attention; the core
    attention is multi-query attention (MQA) with shared key and value.
  * HCA paragraph -- every m' >> m tokens are merged into one entry without
    overlapping compression; no sparse selection, dense attention over the
    compressed entries; both CSA and HCA add a sliding-window attention branch
    over raw recent tokens.
  * storage paragraph -- RoPE dims stored in BF16, the other dims in FP8.

Where the pages are silent this oracle takes the following readings (each is a
choice of this project, stated once here and applied everywhere below):
  R1  compression: per channel c, a softmax over the window positions j of
      (w[c] * x[j,c] + b[j - start, c]), then y[c] = sum_j alpha[j,c] x[j,c].
  R2  CSA windows overlap: entry i covers tokens [(i-1)m, (i+1)m) (2m tokens,
      stride m); HCA entry i covers [i m', (i+1) m').  N = ceil(T / stride).
  R3  window positions outside [0, T) are left out of the softmax, not padded.
  R4  a query at position t sees entry i iff its nominal end (i+1)*stride - 1
      is <= t (a trailing partial entry is therefore never visible).
  R5  the sliding window is the w_s raw tokens [t - w_s + 1, t], t included;
      raw tokens may also be covered by visible entries (double coverage).
  R6  entries and window keys share ONE softmax per query head.
  R7  indexer score s[t,i] = sum_h relu(qI[t,h] . kI[i]) * wI[t,h] (no scale).
  R8  top-k keeps the k highest scores among visible entries, ties to the
      lower index, returned as an ascending set padded with -1.
  R9  "shared key and value": with the FP8/BF16 split cache, V is the
      dequantised 128 non-RoPE channels of the same entry.
  R10 FP8 = OCP E4M3 (bias 7, subnormals, max 448, no infinities), one fp32
      scale per entry = max|x| / 448 (1 when all zero), round to nearest even,
      saturating to +-448.
  R11 the attention also skips selected entries that are out of range or not
      visible (R4), and a query with no keys at all outputs 0 with LSE = -inf.
  R18 FP4 indexer keys (storage paragraph: the lightning indexer in FP4):
      OCP MX E2M1 codes (sign, 2 exponent bits with bias 1, 1 mantissa bit;
      values 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per byte -- dimension 2j in the
      low nibble of byte j, 2j+1 in the high nibble -- and one fp32 scale per
      entry (max|k| / 6, 1 when zero); key = decode(code) * scale.
  R17 grouped output projection: the H heads form G groups of H/G consecutive
      heads; group g's outputs, concatenated head after head, are multiplied
      by the group's own weight W[g] (d_g x (H/G) d_v), giving d_g channels per
      group.  A dense layer that mixes the G groups afterwards is an ordinary
      linear layer outside this method step.
"""
from __future__ import annotations

import math

import numpy as np

D_QK, D_NOPE, D_ROPE, D_V = 192, 128, 64, 128
E4M3_MAX = 448.0


# ----------------------------------------------------------------------------
# entry geometry (R2, R4)
# ----------------------------------------------------------------------------
def n_entries(T: int, stride: int) -> int:
    """Number of compressed entries for T tokens: ceil(T / stride) (R2)."""
    return -(-T // stride)


def entry_start(i: int, stride: int, cwin: int) -> int:
    """First token of entry i's window (may be negative for CSA entry 0)."""
    return i * stride - (cwin - stride)


def entry_end(i: int, stride: int) -> int:
    """Nominal last token of entry i, used for visibility (R4)."""
    return (i + 1) * stride - 1


def n_visible(t: int, stride: int, N: int) -> int:
    """Entries i with entry_end(i) <= t, capped at N."""
    return min(N, (t + 1) // stride)


# ----------------------------------------------------------------------------
# compression (CSA paragraph: learnable weights + position bias; R1-R3)
# ----------------------------------------------------------------------------
def compress(x: np.ndarray, w: np.ndarray, b: np.ndarray, stride: int, cwin: int) -> np.ndarray:
    """Compress raw tokens x [B, T, d] into entries y [B, N, d] (float64).

    CSA: stride m, cwin 2m.  HCA: stride = cwin = m'.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    B, T, d = x.shape
    assert w.shape == (d,) and b.shape == (cwin, d)
    N = n_entries(T, stride)
    y = np.empty((B, N, d), dtype=np.float64)
    for i in range(N):
        s = entry_start(i, stride, cwin)
        j0, j1 = max(s, 0), min(s + cwin, T)          # R3: only in-range tokens
        xs = x[:, j0:j1, :]                            # [B, n, d]
        logit = w[None, None, :] * xs + b[j0 - s:j1 - s, :][None]
        logit = logit - logit.max(axis=1, keepdims=True)
        a = np.exp(logit)
        a = a / a.sum(axis=1, keepdims=True)
        y[:, i, :] = (a * xs).sum(axis=1)
    return y


# ----------------------------------------------------------------------------
# FP8 E4M3 (storage paragraph; R10), written from the OCP OFP8 definition
# ----------------------------------------------------------------------------
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each E4M3 byte: S EEEE MMM, bias 7; E=0 subnormal; S.1111.111 NaN."""
    c = np.asarray(codes, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    mant = (c & 0x7).astype(np.float64)
    normal = s * np.ldexp(1.0 + mant / 8.0, (e - 7).astype(np.int64))
    sub = s * np.ldexp(mant / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((c & 7) == 7), np.nan, v)


_E4M3_POS = e4m3_decode(np.arange(127))     # codes 0x00..0x7E, ascending, 0 .. 448


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round float64 values to E4M3 bytes: nearest, ties to even code, saturate to 448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # first code with value >= a
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    dlo = a - _E4M3_POS[lo]
    dhi = _E4M3_POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(_E4M3_POS[hi] == a, hi, code)
    sign = np.signbit(x).astype(np.int64) << 7          # the sign survives rounding to zero
    return (code | sign).astype(np.uint8)


def e2m1_decode(code4: np.ndarray) -> np.ndarray:
    """Value of each 4-bit E2M1 code S EE M (OCP MX): bias 1; E = 0 subnormal (M * 0.5)."""
    c = np.asarray(code4, dtype=np.int64) & 0xF
    s = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    mant = (c & 0x1).astype(np.float64)
    normal = np.ldexp(1.0 + mant / 2.0, (e - 1).astype(np.int64))
    sub = mant * 0.5
    return s * np.where(e == 0, sub, normal)


def e2m1_unpack(packed: np.ndarray) -> np.ndarray:
    """Bytes [.., d/2] holding two E2M1 codes each -> values [.., d] (dim 2j = low nibble of byte j) (R18)."""
    b = np.asarray(packed, dtype=np.int64)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.float64)
    out[..., 0::2] = e2m1_decode(b & 0xF)
    out[..., 1::2] = e2m1_decode(b >> 4)
    return out


def quantize_entries(y_nope: np.ndarray):
    """Per-entry scale (max|x| / 448, 1 if zero) and E4M3 codes of x / scale (R10)."""
    y = np.asarray(y_nope, dtype=np.float64)
    amax = np.abs(y).max(axis=-1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    codes = e4m3_encode(y / scale[..., None])
    return codes, scale


def dequant_split(codes: np.ndarray, rope: np.ndarray, scale: np.ndarray):
    """Split-cache entries -> (K [.., 192], V [.., 128]) in float64; V = K[..., :128] (R9)."""
    nope = e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]
    k = np.concatenate([nope, np.asarray(rope, dtype=np.float64)], axis=-1)
    return k, nope


# ----------------------------------------------------------------------------
# lightning indexer + top-k (CSA paragraph; R4, R7, R8)
# ----------------------------------------------------------------------------
def indexer_scores(qI: np.ndarray, wI: np.ndarray, kI: np.ndarray, q_pos: np.ndarray,
                   stride: int) -> np.ndarray:
    """s[b, r, i] = sum_h relu(qI[b,r,h] . kI[b,i]) * wI[b,r,h]; -inf where not visible.

    qI [B, R, HI, dI], wI [B, R, HI], kI [B, N, dI], q_pos [R] (positions of the rows).
    """
    qI = np.asarray(qI, dtype=np.float64)
    wI = np.asarray(wI, dtype=np.float64)
    kI = np.asarray(kI, dtype=np.float64)
    B, R, HI, dI = qI.shape
    N = kI.shape[1]
    s = np.empty((B, R, N), dtype=np.float64)
    for bb in range(B):
        dots = np.einsum("rhd,nd->rhn", qI[bb], kI[bb])            # [R, HI, N]
        s[bb] = (np.maximum(dots, 0.0) * wI[bb][:, :, None]).sum(axis=1)
    ends = (np.arange(N) + 1) * stride - 1
    vis = ends[None, :] <= np.asarray(q_pos)[:, None]              # [R, N]
    return np.where(vis[None], s, -np.inf)


def topk_set(s: np.ndarray, k: int) -> np.ndarray:
    """Per row: the k best visible (finite) scores, ties to the lower index.

    Returns int64 [.., k]: the chosen entry indices in ascending order, -1 padded.
    """
    s = np.asarray(s, dtype=np.float64)
    lead = s.shape[:-1]
    flat = s.reshape(-1, s.shape[-1])
    out = np.full((flat.shape[0], k), -1, dtype=np.int64)
    for r in range(flat.shape[0]):
        row = flat[r]
        vis = np.flatnonzero(np.isfinite(row))
        order = np.lexsort((vis, -row[vis]))       # score descending, then index ascending
        chosen = np.sort(vis[order[:k]])
        out[r, :len(chosen)] = chosen
    return out.reshape(*lead, k)


# ----------------------------------------------------------------------------
# core attention: MQA over entries + sliding window, one joint softmax (R5, R6, R11)
# ----------------------------------------------------------------------------
def attend(q_t: np.ndarray, keys: np.ndarray, vals: np.ndarray, scale: float):
    """One query's heads over one shared key/value list (MQA).

    q_t [H, dqk], keys [n, dqk], vals [n, dv] -> (o [H, dv], lse [H], p [H, n]).
    """
    H = q_t.shape[0]
    if keys.shape[0] == 0:
        return np.zeros((H, vals.shape[1])), np.full(H, -np.inf), np.zeros((H, 0))
    logits = scale * (q_t @ keys.T)                      # [H, n]
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    return p @ vals, mx[:, 0] + np.log(l[:, 0]), p


def window_rows(t: int, win_len: int, win_pos0: int, Tw: int) -> np.ndarray:
    """Rows of the raw-token buffer holding positions [max(0, t-win_len+1), t] (R5)."""
    lo = max(0, t - win_len + 1)
    rows = np.arange(lo, t + 1) - win_pos0
    assert win_len == 0 or (rows.size and rows[0] >= 0 and rows[-1] < Tw), \
        "raw-token buffer does not cover the window"
    return rows if win_len > 0 else np.zeros(0, dtype=np.int64)


def _mqa(q, q_pos, Kc, Vc, entry_lists, win_k, win_v, win_pos0, win_len, scale, want_p):
    q = np.asarray(q, dtype=np.float64)
    B, R, H, _ = q.shape
    dv = Vc.shape[-1]
    O = np.zeros((B, R, H, dv))
    LSE = np.zeros((B, R, H))
    P = [] if want_p else None
    Tw = win_k.shape[1]
    for bb in range(B):
        for r in range(R):
            t = int(q_pos[r])
            ent = entry_lists(bb, r, t)
            wr = window_rows(t, win_len, win_pos0, Tw)
            keys = np.concatenate([Kc[bb, ent], win_k[bb, wr]], axis=0)
            vals = np.concatenate([Vc[bb, ent], win_v[bb, wr]], axis=0)
            o, lse, p = attend(q[bb, r], keys, vals, scale)
            O[bb, r], LSE[bb, r] = o, lse
            if want_p:
                P.append(p)
    return (O, LSE, P) if want_p else (O, LSE)


def csa_sparse_mqa(q, q_pos, Kc, Vc, idx, stride, win_k, win_v, win_pos0, win_len, scale,
                   want_p=False):
    """CSA core attention: selected entries idx[b, r, :] (+ window), one softmax.

    q [B, R, H, 192]; Kc [B, N, 192]; Vc [B, N, 128]; idx [B, R, k] (-1 = empty);
    win_k [B, Tw, 192], win_v [B, Tw, 128] hold raw tokens at positions
    win_pos0 .. win_pos0 + Tw - 1.  All float64.
    """
    Kc = np.asarray(Kc, dtype=np.float64)
    Vc = np.asarray(Vc, dtype=np.float64)
    N = Kc.shape[1]
    idx = np.asarray(idx)

    def lists(bb, r, t):
        sel = idx[bb, r]
        ok = (sel >= 0) & (sel < N)
        sel = sel[ok]
        return sel[(sel + 1) * stride - 1 <= t]          # R11: visible entries only

    return _mqa(q, q_pos, Kc, Vc, lists, np.asarray(win_k, np.float64), np.asarray(win_v, np.float64),
                win_pos0, win_len, scale, want_p)


def hca_dense_mqa(q, q_pos, Kc, Vc, stride, win_k, win_v, win_pos0, win_len, scale, want_p=False):
    """HCA core attention: every visible entry (+ window), one softmax."""
    Kc = np.asarray(Kc, dtype=np.float64)
    Vc = np.asarray(Vc, dtype=np.float64)
    N = Kc.shape[1]

    def lists(bb, r, t):
        return np.arange(n_visible(t, stride, N))

    return _mqa(q, q_pos, Kc, Vc, lists, np.asarray(win_k, np.float64), np.asarray(win_v, np.float64),
                win_pos0, win_len, scale, want_p)


# ----------------------------------------------------------------------------
# grouped output projection (CSA paragraph: the MQA is followed by a grouped
# output projection that keeps its cost down; R17)
# ----------------------------------------------------------------------------
def grouped_out_proj(o: np.ndarray, W: np.ndarray) -> np.ndarray:
    """y[.., g, :] = concat_{h in group g} o[.., h, :]  @  W[g]^T   (float64).

    o [.., H, dv]: attention outputs; W [G, d_g, (H/G) * dv]: row j of W[g] holds the
    weights of group g's output channel j.  Returns y [.., G, d_g].
    """
    o = np.asarray(o, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    G, dg, K = W.shape
    H, dv = o.shape[-2], o.shape[-1]
    hg = H // G
    assert H % G == 0 and K == hg * dv, "W must be [G, d_g, (H/G) * dv]"
    lead = o.shape[:-2]
    y = np.empty(lead + (G, dg), dtype=np.float64)
    for g in range(G):
        x = o[..., g * hg:(g + 1) * hg, :].reshape(lead + (K,))   # head g*hg first, then the next
        y[..., g, :] = x @ W[g].T
    return y


def default_scale(d_qk: int = D_QK) -> float:
    return 1.0 / math.sqrt(d_qk)
