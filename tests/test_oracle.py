"""Pins for the CPU oracle: closed forms, invariants, special cases and brute force.

Each test checks the oracle against something other than its own formula, so a
dropped term, a wrong sign or index, or a transposed operand fails at least one
of them.  CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import csa_ref as R

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


# ---------------------------------------------------------------------------
# compression
# ---------------------------------------------------------------------------
def test_compress_window_one_is_identity():
    x = rng.standard_normal((2, 9, 5))
    y = R.compress(x, rng.standard_normal(5), rng.standard_normal((1, 5)), stride=1, cwin=1)
    assert np.array_equal(y, x)


@pytest.mark.parametrize("T,m,cwin", [(13, 4, 8), (16, 4, 8), (10, 3, 3), (7, 8, 16)])
def test_compress_zero_params_is_window_mean(T, m, cwin):
    x = rng.standard_normal((2, T, 3))
    y = R.compress(x, np.zeros(3), np.zeros((cwin, 3)), m, cwin)
    N = -(-T // m)
    assert y.shape == (2, N, 3)
    for i in range(N):
        lo = max(0, i * m - (cwin - m))
        hi = min(T, i * m - (cwin - m) + cwin)
        np.testing.assert_allclose(y[:, i], x[:, lo:hi].mean(axis=1), rtol=0, atol=1e-14)
    if cwin == 2 * m:      # CSA entry 0 averages only its m in-range tokens
        np.testing.assert_allclose(y[:, 0], x[:, :m].mean(axis=1), atol=1e-14)


def test_compress_two_token_window_is_sigmoid_mix():
    # stride 1, window 2, w = 0: entry i >= 1 mixes x[i-1], x[i] with weights
    # sigmoid(b0 - b1), sigmoid(b1 - b0); entry 0 has only x[0] in range.
    x = rng.standard_normal((1, 6, 4))
    b = rng.standard_normal((2, 4))
    y = R.compress(x, np.zeros(4), b, stride=1, cwin=2)
    sig = 1.0 / (1.0 + np.exp(-(b[0] - b[1])))
    np.testing.assert_allclose(y[0, 0], x[0, 0], atol=1e-15)
    for i in range(1, 6):
        np.testing.assert_allclose(y[0, i], sig * x[0, i - 1] + (1 - sig) * x[0, i], atol=1e-14)


def test_compress_convex_and_bias_shift_invariant():
    x = rng.standard_normal((2, 37, 6))
    w = rng.standard_normal(6)
    b = rng.standard_normal((8, 6))
    y = R.compress(x, w, b, 4, 8)
    y2 = R.compress(x, w, b + rng.standard_normal(6)[None, :] * 5, 4, 8)
    np.testing.assert_allclose(y, y2, atol=1e-12)
    for i in range(y.shape[1]):
        lo, hi = max(0, (i - 1) * 4), min(37, (i + 1) * 4)
        seg = x[:, lo:hi]
        assert np.all(y[:, i] <= seg.max(axis=1) + 1e-12)
        assert np.all(y[:, i] >= seg.min(axis=1) - 1e-12)


def test_compress_large_weight_selects_extremes():
    T, d = 24, 5
    base = np.stack([rng.permutation(T) * 0.1 for _ in range(d)], axis=1)[None]   # distinct values
    yp = R.compress(base, np.full(d, 1e4), np.zeros((8, d)), 4, 8)
    yn = R.compress(base, np.full(d, -1e4), np.zeros((8, d)), 4, 8)
    for i in range(T // 4):
        lo, hi = max(0, (i - 1) * 4), (i + 1) * 4
        np.testing.assert_allclose(yp[0, i], base[0, lo:hi].max(axis=0), atol=1e-12)
        np.testing.assert_allclose(yn[0, i], base[0, lo:hi].min(axis=0), atol=1e-12)


def test_compress_position_bias_indexes_window_offset():
    # a huge bias at window offset o makes entry i copy token start_i + o,
    # unless that token is out of range (then the bias is simply not used).
    T, m, d = 20, 4, 3
    x = rng.standard_normal((1, T, d))
    for o in range(8):
        b = np.zeros((8, d))
        b[o] = 1e4
        y = R.compress(x, np.zeros(d), b, m, 8)
        for i in range(T // m):
            j = (i - 1) * m + o
            if 0 <= j < T:
                np.testing.assert_allclose(y[0, i], x[0, j], atol=1e-12)
            else:   # only entry 0 (offsets 0..m-1 before the sequence)
                assert i == 0 and o < m
                np.testing.assert_allclose(y[0, 0], x[0, :m].mean(axis=0), atol=1e-12)


@pytest.mark.parametrize("T,N", [(8192, 64), (8191, 64), (1000, 8), (128, 1), (129, 2)])
def test_hca_entry_count(T, N):
    x = rng.standard_normal((1, T, 2))
    assert R.compress(x, np.zeros(2), np.zeros((128, 2)), 128, 128).shape[1] == N
    assert R.n_entries(T, 128) == N


def test_compress_token_reach():
    # token j feeds CSA entries floor(j/m) and floor(j/m)+1 only; HCA entry floor(j/m') only
    T, m, d = 32, 4, 2
    x = rng.standard_normal((1, T, d))
    w, b = rng.standard_normal(d), rng.standard_normal((8, d))
    base = R.compress(x, w, b, m, 8)
    for j in range(T):
        x2 = x.copy()
        x2[0, j] += 1.0
        changed = np.flatnonzero(np.any(R.compress(x2, w, b, m, 8)[0] != base[0], axis=1))
        expect = [i for i in (j // m, j // m + 1) if i < T // m]
        assert list(changed) == expect
    hb = R.compress(x, w, b[:m], m, m)
    for j in range(T):
        x2 = x.copy()
        x2[0, j] += 1.0
        changed = np.flatnonzero(np.any(R.compress(x2, w, b[:m], m, m)[0] != hb[0], axis=1))
        assert list(changed) == [j // m]


# ---------------------------------------------------------------------------
# FP8 E4M3
# ---------------------------------------------------------------------------
def _golden_e4m3():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_ocp_values.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                c, v = line.split()
                rows.append((int(c, 16), float(v)))
    return rows


def test_e4m3_golden_values():
    rows = _golden_e4m3()
    vals = R.e4m3_decode(np.array([c for c, _ in rows]))
    for (c, v), got in zip(rows, vals):
        if math.isnan(v):
            assert math.isnan(got), hex(c)
        else:
            assert got == v and math.copysign(1, got) == math.copysign(1, v), hex(c)


def test_e4m3_decode_matches_torch_for_all_codes():
    c = np.arange(256, dtype=np.uint8)
    t = torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()
    v = R.e4m3_decode(c)
    assert np.array_equal(np.isnan(v), np.isnan(t))
    ok = ~np.isnan(v)
    assert np.array_equal(v[ok], t[ok])


def test_e4m3_encode_matches_torch_rne():
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 1, 30, 300)])
    vals = R.e4m3_decode(np.arange(127))
    mids = (vals[:-1] + vals[1:]) / 2                       # exact ties
    x = np.concatenate([x, mids, -mids, [0.0, 448.0, 500.0, -1e9]])
    ours = R.e4m3_encode(x)
    lib = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)
    # ties go to the even code
    assert np.all(R.e4m3_encode(mids) % 2 == 0)


def test_e4m3_round_trip_and_half_ulp():
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    assert np.array_equal(R.e4m3_encode(R.e4m3_decode(finite)), finite.astype(np.uint8))
    x = rng.standard_normal((64, 128)) * 3
    codes, scale = R.quantize_entries(x)
    back = R.e4m3_decode(codes) * scale[:, None]
    # half an ulp of the E4M3 grid at each value's binade (subnormal spacing 2^-9)
    a = np.abs(x / scale[:, None])
    ulp = np.where(a < 2 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(a, 2 ** -6))) - 3))
    assert np.all(np.abs(back - x) <= 0.5 * ulp * scale[:, None] * (1 + 1e-12))
    assert np.all(np.abs(R.e4m3_decode(codes)).max(axis=1) == 448.0)


# ---------------------------------------------------------------------------
# indexer + top-k
# ---------------------------------------------------------------------------
def _brute_topk(row, k):
    cand = [i for i in range(len(row)) if np.isfinite(row[i])]
    best = sorted(cand, key=lambda i: (-row[i], i))[:k]
    return sorted(best) + [-1] * (k - len(best))


def test_topk_brute_force_random_and_ties():
    for trial in range(30):
        n = int(rng.integers(1, 60))
        k = int(rng.integers(1, 70))
        row = rng.integers(-3, 4, n).astype(np.float64)      # many exact ties
        row[rng.random(n) < 0.2] = -np.inf
        assert list(R.topk_set(row[None], k)[0]) == _brute_topk(row, k)
        row = rng.standard_normal(n)
        assert list(R.topk_set(row[None], k)[0]) == _brute_topk(row, k)


def test_indexer_single_head_single_dim_closed_form():
    # wI = (1,0,0,0) and qI head 0 = unit vector e_j: s[t,i] = relu(kI[i, j])
    B, T, N, m = 1, 4, 10, 1
    kI = rng.standard_normal((B, N, 64))
    qI = np.zeros((B, T, 4, 64))
    qI[0, :, 0, 5] = 1.0
    qI[0, :, 1:, :] = rng.standard_normal((T, 3, 64))
    wI = np.zeros((B, T, 4))
    wI[..., 0] = 1.0
    pos = np.array([N - 1] * T)
    s = R.indexer_scores(qI, wI, kI, pos, m)
    np.testing.assert_allclose(s[0, 0], np.maximum(kI[0, :, 5], 0), atol=1e-15)


def test_indexer_weights_each_head_and_relu():
    # two heads with opposite queries: exactly one of them is positive per entry
    N = 16
    kI = rng.standard_normal((1, N, 64))
    u = rng.standard_normal(64)
    qI = np.zeros((1, 1, 4, 64))
    qI[0, 0, 0], qI[0, 0, 1] = u, -u
    wI = np.array([[[2.0, 3.0, 0.0, 0.0]]])
    s = R.indexer_scores(qI, wI, kI, np.array([10 ** 6]), 4)[0, 0]
    d = kI[0] @ u
    np.testing.assert_allclose(s, np.where(d > 0, 2 * d, -3 * d), atol=1e-12)


def test_indexer_visibility_and_all_visible_set():
    m, N = 4, 12
    kI = rng.standard_normal((1, N, 64))
    qI = rng.standard_normal((1, 50, 4, 64))
    wI = rng.random((1, 50, 4))
    pos = np.arange(50)
    s = R.indexer_scores(qI, wI, kI, pos, m)
    idx = R.topk_set(s, 64)
    for t in range(50):
        nv = min(N, (t + 1) // m)
        assert np.isfinite(s[0, t]).sum() == nv
        assert list(idx[0, t, :nv]) == list(range(nv)) and np.all(idx[0, t, nv:] == -1)


def test_indexer_planted_maxima_and_tie_rule():
    N, k = 40, 5
    u = rng.standard_normal(64)
    kI = rng.standard_normal((1, N, 64)) * 0.01
    planted = [3, 17, 18, 30, 39]
    for j, i in enumerate(planted):
        kI[0, i] = u * (10 + j)
    qI = np.tile(u, (1, 1, 4, 1))
    wI = rng.random((1, 1, 4)) + 0.5
    s = R.indexer_scores(qI, wI, kI, np.array([4 * N]), 4)
    assert list(R.topk_set(s, k)[0, 0]) == planted
    # exact ties: entries 7 and 2 get the same key; k=1 must pick the lower index
    kI2 = kI.copy()
    kI2[0, 2] = kI2[0, 7] = u * 100
    s2 = R.indexer_scores(qI, wI, kI2, np.array([4 * N]), 4)
    assert list(R.topk_set(s2, 1)[0, 0]) == [2]
    # positive rescaling of the head weights keeps the set
    s3 = R.indexer_scores(qI, wI * 3.7, kI, np.array([4 * N]), 4)
    assert np.array_equal(R.topk_set(s3, 7), R.topk_set(s, 7))


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def _textbook_causal_mqa(q, K, V, scale, bonus_last=0, bonus=0.0):
    """Full-matrix masked softmax attention; optional +bonus on the last keys."""
    B, T, H, _ = q.shape
    O = np.zeros((B, T, H, V.shape[-1]))
    for b in range(B):
        S = scale * np.einsum("thd,jd->thj", q[b], K[b])
        t_idx = np.arange(T)[:, None]
        j_idx = np.arange(T)[None, :]
        mask = j_idx <= t_idx
        extra = np.where((j_idx <= t_idx) & (j_idx > t_idx - bonus_last), bonus, 0.0)
        S = np.where(mask[:, None, :], S + extra[:, None, :], -np.inf)
        P = np.exp(S - S.max(axis=2, keepdims=True))
        P /= P.sum(axis=2, keepdims=True)
        O[b] = np.einsum("thj,jd->thd", P, V[b])
    return O


def _dense_special_case(win_len):
    B, T, H = 2, 11, 3
    q = rng.standard_normal((B, T, H, 192))
    K = rng.standard_normal((B, T, 192))
    V = rng.standard_normal((B, T, 128))
    Kc = R.compress(K, rng.standard_normal(192), rng.standard_normal((1, 192)), 1, 1)
    Vc = R.compress(V, rng.standard_normal(128), rng.standard_normal((1, 128)), 1, 1)
    idx = np.tile(np.arange(T), (B, T, 1))                 # k >= N: everything selected
    sc = 0.1
    O, _ = R.csa_sparse_mqa(q, np.arange(T), Kc, Vc, idx, 1, K, V, 0, win_len, sc)
    return O, q, K, V, sc


def test_csa_m1_full_selection_no_window_is_dense_causal_mqa():
    O, q, K, V, sc = _dense_special_case(0)
    np.testing.assert_allclose(O, _textbook_causal_mqa(q, K, V, sc), atol=1e-12)


@pytest.mark.parametrize("w", [1, 4, 64])
def test_window_double_coverage_is_ln2_bonus(w):
    O, q, K, V, sc = _dense_special_case(w)
    np.testing.assert_allclose(O, _textbook_causal_mqa(q, K, V, sc, bonus_last=w, bonus=math.log(2)),
                               atol=1e-12)


def _mask_matrix_csa(q, Kc, Vc, idx, m, K, V, win_len, scale):
    """Second formulation: one [T, N + T] mask per sequence, softmax over the full row."""
    B, T, H, _ = q.shape
    N = Kc.shape[1]
    O = np.zeros((B, T, H, V.shape[-1]))
    for b in range(B):
        keys = np.concatenate([Kc[b], K[b]])
        vals = np.concatenate([Vc[b], V[b]])
        mask = np.zeros((T, N + T), dtype=bool)
        for t in range(T):
            for i in idx[b, t]:
                if 0 <= i < N and (i + 1) * m - 1 <= t:
                    mask[t, i] = True
            mask[t, N + max(0, t - win_len + 1):N + t + 1] = True
        S = scale * np.einsum("thd,jd->thj", q[b], keys)
        S = np.where(mask[:, None, :], S, -np.inf)
        P = np.exp(S - S.max(axis=2, keepdims=True))
        O[b] = np.einsum("thj,jd->thd", P / P.sum(axis=2, keepdims=True), vals)
    return O


def _small_csa(B=2, T=37, H=4, m=4, k=5, win=6, seed=0):
    g = np.random.default_rng(seed)
    x = dict(q=_bf16(g.standard_normal((B, T, H, 192))), K=_bf16(g.standard_normal((B, T, 192))),
             V=_bf16(g.standard_normal((B, T, 128))), qI=_bf16(g.standard_normal((B, T, 4, 64))),
             kI=_bf16(g.standard_normal((B, T, 64))), wI=g.random((B, T, 4)),
             wk=g.standard_normal(192) * 0.02, bk=g.standard_normal((2 * m, 192)) * 0.1,
             wv=g.standard_normal(128) * 0.02, bv=g.standard_normal((2 * m, 128)) * 0.1,
             wi=g.standard_normal(64) * 0.02, bi=g.standard_normal((2 * m, 64)) * 0.1)
    return x


def _run_csa(x, m, k, win, scale=1 / math.sqrt(192)):
    T = x["q"].shape[1]
    Kc = R.compress(x["K"], x["wk"], x["bk"], m, 2 * m)
    Vc = R.compress(x["V"], x["wv"], x["bv"], m, 2 * m)
    kIc = R.compress(x["kI"], x["wi"], x["bi"], m, 2 * m)
    s = R.indexer_scores(x["qI"], x["wI"], kIc, np.arange(T), m)
    idx = R.topk_set(s, k)
    O, L, P = R.csa_sparse_mqa(x["q"], np.arange(T), Kc, Vc, idx, m, x["K"], x["V"], 0, win, scale,
                               want_p=True)
    return O, L, P, idx, Kc, Vc


def test_csa_loop_oracle_equals_mask_matrix_form():
    x = _small_csa()
    O, _, _, idx, Kc, Vc = _run_csa(x, 4, 5, 6)
    O2 = _mask_matrix_csa(x["q"], Kc, Vc, idx, 4, x["K"], x["V"], 6, 1 / math.sqrt(192))
    np.testing.assert_allclose(O, O2, atol=1e-12)


def test_softmax_weights_sum_to_one():
    x = _small_csa()
    _, _, P, _, _, _ = _run_csa(x, 4, 5, 6)
    for p in P:
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)


def test_joint_softmax_equals_lse_merge_of_branches():
    # the two key sets share one softmax: merging per-branch results by their
    # log-sum-exp must give the joint result (and not e.g. their average)
    x = _small_csa(B=1, T=30)
    m, k, win = 4, 3, 5
    T = 30
    Kc = R.compress(x["K"], x["wk"], x["bk"], m, 8)
    Vc = R.compress(x["V"], x["wv"], x["bv"], m, 8)
    kIc = R.compress(x["kI"], x["wi"], x["bi"], m, 8)
    idx = R.topk_set(R.indexer_scores(x["qI"], x["wI"], kIc, np.arange(T), m), k)
    sc = 0.07
    Oj, Lj = R.csa_sparse_mqa(x["q"], np.arange(T), Kc, Vc, idx, m, x["K"], x["V"], 0, win, sc)
    Oe, Le = R.csa_sparse_mqa(x["q"], np.arange(T), Kc, Vc, idx, m, x["K"], x["V"], 0, 0, sc)
    Ow, Lw = R.csa_sparse_mqa(x["q"], np.arange(T), Kc, Vc, np.full_like(idx, -1), m,
                              x["K"], x["V"], 0, win, sc)
    L = np.logaddexp(Le, Lw)
    we, ww = np.exp(Le - L), np.exp(Lw - L)
    Om = np.nan_to_num(we)[..., None] * Oe + ww[..., None] * Ow
    np.testing.assert_allclose(Oj, Om, atol=1e-12)
    np.testing.assert_allclose(Lj, L, atol=1e-12)


def test_causality_perturbing_future_changes_nothing():
    m, k, win = 4, 5, 6
    x = _small_csa(B=1, T=41)
    O, _, _, _, _, _ = _run_csa(x, m, k, win)
    for t in (0, 3, 4, 17, 30):
        y = {kk: (v.copy() if isinstance(v, np.ndarray) else v) for kk, v in x.items()}
        for name in ("q", "K", "V", "qI", "kI", "wI"):
            y[name][:, t + 1:] = rng.standard_normal(y[name][:, t + 1:].shape) * 3
        O2, _, _, _, _, _ = _run_csa(y, m, k, win)
        assert np.array_equal(O[:, :t + 1], O2[:, :t + 1])
    # HCA too
    mp = 8
    xq, xK, xV = x["q"], x["K"], x["V"]
    Kc = R.compress(xK, x["wk"], np.zeros((mp, 192)), mp, mp)
    Vc = R.compress(xV, x["wv"], np.zeros((mp, 128)), mp, mp)
    O, _ = R.hca_dense_mqa(xq, np.arange(41), Kc, Vc, mp, xK, xV, 0, win, 0.1)
    for t in (5, 7, 8, 20):
        K2, V2 = xK.copy(), xV.copy()
        K2[:, t + 1:] += 1.0
        V2[:, t + 1:] -= 2.0
        Kc2 = R.compress(K2, x["wk"], np.zeros((mp, 192)), mp, mp)
        Vc2 = R.compress(V2, x["wv"], np.zeros((mp, 128)), mp, mp)
        O2, _ = R.hca_dense_mqa(xq, np.arange(41), Kc2, Vc2, mp, K2, V2, 0, win, 0.1)
        assert np.array_equal(O[:, :t + 1], O2[:, :t + 1])


def test_hca_equals_csa_selecting_everything():
    B, T, H, mp, win = 2, 70, 3, 16, 9
    q = rng.standard_normal((B, T, H, 192))
    K = rng.standard_normal((B, T, 192))
    V = rng.standard_normal((B, T, 128))
    Kc = R.compress(K, rng.standard_normal(192), rng.standard_normal((mp, 192)), mp, mp)
    Vc = R.compress(V, rng.standard_normal(128), rng.standard_normal((mp, 128)), mp, mp)
    N = Kc.shape[1]
    idx = np.tile(np.arange(N), (B, T, 1))
    O1, L1 = R.hca_dense_mqa(q, np.arange(T), Kc, Vc, mp, K, V, 0, win, 0.2)
    O2, L2 = R.csa_sparse_mqa(q, np.arange(T), Kc, Vc, idx, mp, K, V, 0, win, 0.2)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(L1, L2, atol=1e-13)


def test_window_covers_every_token_not_in_a_visible_entry():
    # with w_s >= stride every token <= t is covered by a visible entry or the window
    for stride, cwin, ws in ((4, 8, 128), (128, 128, 128), (4, 8, 4)):
        for t in range(0, 600, 7):
            nv = (t + 1) // stride
            covered = set()
            for i in range(nv):
                covered.update(range(max(0, i * stride - (cwin - stride)), (i + 1) * stride))
            covered.update(range(max(0, t - ws + 1), t + 1))
            assert covered == set(range(t + 1))


def test_decode_equals_last_prefill_row_with_shared_kv():
    # V := K[:, :128] for raw tokens and for entries; a decode query at t = T-1
    # over the cache + the last w_s raw tokens equals the prefill's last row.
    g = np.random.default_rng(7)
    B, T, H, m, k, win = 2, 64, 4, 4, 6, 10
    q = g.standard_normal((B, T, H, 192))
    K = g.standard_normal((B, T, 192))
    wk, bk = g.standard_normal(192) * 0.02, g.standard_normal((8, 192)) * 0.1
    Kc = R.compress(K, wk, bk, m, 8)
    Vc = Kc[..., :128]
    kIc = g.standard_normal((B, T // m, 64))
    qI, wI = g.standard_normal((B, T, 4, 64)), g.random((B, T, 4))
    idx = R.topk_set(R.indexer_scores(qI, wI, kIc, np.arange(T), m), k)
    Op, Lp = R.csa_sparse_mqa(q, np.arange(T), Kc, Vc, idx, m, K, K[..., :128], 0, win, 0.1)
    idx_d = R.topk_set(R.indexer_scores(qI[:, -1:], wI[:, -1:], kIc, np.array([T - 1]), m), k)
    assert np.array_equal(idx_d[:, 0], idx[:, -1])
    wk_ = K[:, T - win:]
    Od, Ld = R.csa_sparse_mqa(q[:, -1:], np.array([T - 1]), Kc, Vc, idx_d, m, wk_, wk_[..., :128],
                              T - win, win, 0.1)
    np.testing.assert_allclose(Od[:, 0], Op[:, -1], atol=1e-13)
    np.testing.assert_allclose(Ld[:, 0], Lp[:, -1], atol=1e-13)


def test_split_cache_dequant_shares_k_and_v():
    codes = rng.integers(0, 256, (3, 5, 128)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x10
    rope = rng.standard_normal((3, 5, 64))
    scale = rng.random((3, 5)) + 0.1
    K, V = R.dequant_split(codes, rope, scale)
    assert K.shape == (3, 5, 192) and V.shape == (3, 5, 128)
    assert np.array_equal(K[..., :128], V)
    assert np.array_equal(K[..., 128:], rope)
    np.testing.assert_allclose(V[1, 2, 3], R.e4m3_decode(codes[1, 2, 3]) * scale[1, 2], rtol=0)


# ---------------------------------------------------------------------------
# grouped output projection (R17)
# ---------------------------------------------------------------------------
def test_grouped_out_proj_is_block_diagonal_dense_projection():
    """The grouped projection equals one dense projection of the flattened heads by the
    block-diagonal matrix whose diagonal blocks are the groups' weights (scipy builds it)."""
    from scipy.linalg import block_diag
    R_, H, dv, G, dg = 5, 8, 6, 4, 7
    o = rng.standard_normal((R_, H, dv))
    W = rng.standard_normal((G, dg, (H // G) * dv))
    y = R.grouped_out_proj(o, W)
    dense = block_diag(*[W[g].T for g in range(G)])          # [(H*dv), (G*dg)]
    assert dense.shape == (H * dv, G * dg)
    np.testing.assert_allclose(y.reshape(R_, G * dg), o.reshape(R_, H * dv) @ dense, rtol=1e-12, atol=1e-12)


def test_grouped_out_proj_selector_weights_pick_channels():
    """Weights that select one channel: output j of group g reads head g*hg + (j % hg), channel j."""
    H, dv, G, dg = 6, 5, 3, 4
    hg = H // G
    W = np.zeros((G, dg, hg * dv))
    for g in range(G):
        for j in range(dg):
            W[g, j, (j % hg) * dv + j] = 1.0
    o = rng.standard_normal((2, 3, H, dv))
    y = R.grouped_out_proj(o, W)
    for g in range(G):
        for j in range(dg):
            assert np.array_equal(y[..., g, j], o[..., g * hg + j % hg, j])


def test_grouped_out_proj_one_head_per_group_identity():
    H, dv = 4, 3
    o = rng.standard_normal((7, H, dv))
    W = np.stack([np.eye(dv)] * H)                            # G = H groups of one head, W_g = I
    assert np.array_equal(R.grouped_out_proj(o, W), o)


# ---------------------------------------------------------------------------
# FP4 E2M1 indexer keys (R18)
# ---------------------------------------------------------------------------
def test_e2m1_golden_values():
    rows = []
    for line in open(os.path.join(GOLDEN, "e2m1_ocp_values.txt")):
        if line.strip() and not line.startswith("#"):
            c, v = line.split()
            rows.append((int(c, 16), float(v)))
    assert len(rows) == 16
    codes = np.array([c for c, _ in rows])
    vals = R.e2m1_decode(codes)
    for (c, v), got in zip(rows, vals):
        assert got == v and np.signbit(got) == np.signbit(v), (hex(c), got, v)


def test_e2m1_unpack_nibble_order():
    """Dimension 2j sits in the low nibble of byte j: the byte 0x72 holds (1.0, 6.0) in that order."""
    packed = np.array([[0x72, 0xA9, 0x0F]], dtype=np.uint8)
    assert R.e2m1_unpack(packed).tolist() == [[1.0, 6.0, -0.5, -1.0, -6.0, 0.0]]


def test_e2m1_values_are_the_grid_between_adjacent_powers():
    """Every nonzero magnitude is 2^e * (1 + m/2) for e in {0, 1, 2} or the subnormal 0.5, and the set
    {0, 0.5, 1, 1.5, 2, 3, 4, 6} is symmetric under the sign bit."""
    v = R.e2m1_decode(np.arange(16))
    assert sorted(set(np.abs(v).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(v[8:], -v[:8])
