"""GPU parity of the incremental cache append and of packed (variable-length)
sequences against the float64 oracle, which handles every sequence on its own.

Append: the entry a decode token completes equals the oracle's entry of the
whole sequence (FP8 epilogue rule for the split cache), nothing else in the
cache changes, and appending at every step reproduces the full compression.
Packed: each sequence's entries equal the oracle's compression of that
sequence alone (no window reaches into a neighbour)."""
import numpy as np
import pytest
import torch

import long_context_sparse_10_b200 as csa
from oracle import csa_ref as R
from parity import assert_close, assert_lse, check_topk, e4m3_ordinal, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16(g, shape, std=1.0):
    return torch.from_numpy((g.standard_normal(shape) * std).astype(np.float32)).to(torch.bfloat16)


def _f32(g, shape, std):
    return torch.from_numpy((g.standard_normal(shape) * std).astype(np.float32))


@pytest.mark.parametrize("kind,m,t", [("csa", 4, 4 * 700 + 3), ("csa", 4, 3), ("hca", 128, 128 * 40 + 127),
                                      ("hca", 128, 127)])
def test_append_split_fp8_matches_oracle_entry(kind, m, t):
    g = np.random.default_rng(t + m)
    B, d, n_cap = 3, 192, 800 if kind == "csa" else 64
    cw = 2 * m if kind == "csa" else m
    X = _bf16(g, (B, t + 1, d))                        # the whole sequence so far
    w, b = _f32(g, (d,), 0.02), _f32(g, (cw, d), 0.1)
    rows = 256
    x_pos0 = max(0, t + 1 - rows)
    xbuf = X[:, x_pos0:].contiguous()                   # the recent raw tokens the decoder keeps
    nope = torch.full((B, n_cap, 128), 0x5A, dtype=torch.uint8, device=DEV)
    rope = torch.full((B, n_cap, 64), 3.0, dtype=torch.bfloat16, device=DEV)
    scale = torch.full((B, n_cap), -1.0, dtype=torch.float32, device=DEV)
    cache = csa.KVCache(nope=nope, rope=rope, scale=scale)
    fn = csa.csa_compress_append if kind == "csa" else csa.hca_compress_append
    fn(xbuf.to(DEV), x_pos0, t, w.to(DEV), b.to(DEV), m, cache)
    torch.cuda.synchronize()
    i = (t + 1) // m - 1
    y = R.compress(f64(X), f64(w), f64(b), m, cw)[:, i]
    codes, sc = R.quantize_entries(y[:, :128])
    np.testing.assert_allclose(scale[:, i].cpu().numpy(), sc, rtol=1e-5)
    dd = np.abs(e4m3_ordinal(nope[:, i].cpu().numpy()) - e4m3_ordinal(codes))
    assert dd.max() <= 1
    assert_close(f64(rope[:, i]), y[:, 128:], "appended rope")
    others = np.ones(n_cap, bool)
    others[i] = False
    assert (nope[:, others] == 0x5A).all() and (scale[:, others] == -1.0).all() and (rope[:, others] == 3.0).all()


def test_append_between_stride_boundaries_does_nothing():
    g = np.random.default_rng(1)
    lib = csa._lib.load()
    x = _bf16(g, (2, 16, 64)).to(DEV)
    cache = torch.zeros(2, 10, 64, dtype=torch.bfloat16, device=DEV)
    before = lib.csa_launch_count()
    csa.csa_compress_append(x, 0, 13, torch.zeros(64, device=DEV), torch.zeros(8, 64, device=DEV), 4, cache)
    torch.cuda.synchronize()
    assert lib.csa_launch_count() == before and torch.count_nonzero(cache) == 0


@pytest.mark.parametrize("kind,m,d", [("csa", 4, 192), ("csa", 4, 64), ("hca", 16, 128)])
def test_append_every_step_reproduces_full_compression(kind, m, d):
    """A decode loop that appends after every token builds exactly (bit for bit) the cache that compressing
    the whole sequence at once gives."""
    g = np.random.default_rng(7 + d)
    B, T = 2, 203
    cw = 2 * m if kind == "csa" else m
    X = _bf16(g, (B, T, d)).to(DEV)
    w, b = _f32(g, (d,), 0.02).to(DEV), _f32(g, (cw, d), 0.1).to(DEV)
    full = (csa.csa_compress if kind == "csa" else csa.hca_compress)(X, w, b, m)
    n_cap = full.shape[1]
    cache = torch.zeros(B, n_cap, d, dtype=torch.bfloat16, device=DEV)
    fn = csa.csa_compress_append if kind == "csa" else csa.hca_compress_append
    rows = 2 * cw
    for t in range(T):
        x0 = max(0, t + 1 - rows)
        fn(X[:, x0:t + 1].contiguous(), x0, t, w, b, m, cache)
    torch.cuda.synchronize()
    complete = T // m                                   # the trailing partial entry never completes
    assert torch.equal(cache[:, :complete], full[:, :complete])


@pytest.mark.parametrize("kind,m,d,fp8", [("csa", 4, 192, False), ("csa", 4, 192, True), ("csa", 4, 64, False),
                                          ("hca", 128, 128, False), ("hca", 32, 192, True)])
def test_packed_compression_is_per_sequence(kind, m, d, fp8):
    g = np.random.default_rng(m + d + fp8)
    lens = [37, 1, 300, 8, 0, 129, 4]
    pk = csa.Packed(lens, m)
    cw = 2 * m if kind == "csa" else m
    x = _bf16(g, (pk.total_tokens, d))
    w, b = _f32(g, (d,), 0.02), _f32(g, (cw, d), 0.1)
    fn = csa.csa_compress_packed if kind == "csa" else csa.hca_compress_packed
    out = fn(x.to(DEV), pk, w.to(DEV), b.to(DEV), m, fp8=fp8)
    torch.cuda.synchronize()
    for s, n in enumerate(lens):
        t0, e0, e1 = pk.cu_tokens_host[s], pk.cu_entries_host[s], pk.cu_entries_host[s + 1]
        if n == 0:
            assert e1 == e0
            continue
        y = R.compress(f64(x[t0:t0 + n])[None], f64(w), f64(b), m, cw)[0]
        assert y.shape[0] == e1 - e0
        if fp8:
            nope, rope, scale = out
            codes, sc = R.quantize_entries(y[:, :128])
            np.testing.assert_allclose(scale[e0:e1].cpu().numpy(), sc, rtol=1e-5)
            assert np.abs(e4m3_ordinal(nope[e0:e1].cpu().numpy()) - e4m3_ordinal(codes)).max() <= 1
            assert_close(f64(rope[e0:e1]), y[:, 128:], f"packed rope seq {s}")
        else:
            assert_close(f64(out[e0:e1]), y, f"packed {kind} seq {s}")


def _round_bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("H,lens,k,win", [
    (16, [300, 1, 64, 1000, 7, 513], 64, 128),
    (64, [700, 3, 1300, 260], 128, 128),
])
def test_packed_csa_prefill_pipeline_is_per_sequence(H, lens, k, win):
    """Packed CSA prefill (compress -> indexer top-k -> sparse MQA): every sequence equals the oracle
    pipeline run on that sequence alone -- no window, score or attention crosses a sequence boundary."""
    g = np.random.default_rng(H + len(lens))
    m = 4
    pk = csa.Packed(lens, m)
    TT = pk.total_tokens
    q, K, V = _bf16(g, (TT, H, 192)), _bf16(g, (TT, 192)), _bf16(g, (TT, 128))
    qI, kI = _bf16(g, (TT, 4, 64)), _bf16(g, (TT, 64))
    wI = torch.from_numpy(g.random((TT, 4)).astype(np.float32))
    wk, bk, wv, bv = _f32(g, (192,), 0.02), _f32(g, (8, 192), 0.1), _f32(g, (128,), 0.02), _f32(g, (8, 128), 0.1)
    wi, bi = _f32(g, (64,), 0.02), _f32(g, (8, 64), 0.1)
    d = {n: t.to(DEV) for n, t in dict(q=q, K=K, V=V, qI=qI, kI=kI, wI=wI, wk=wk, bk=bk, wv=wv, bv=bv, wi=wi,
                                       bi=bi).items()}
    Kc = csa.csa_compress_packed(d["K"], pk, d["wk"], d["bk"], m)
    Vc = csa.csa_compress_packed(d["V"], pk, d["wv"], d["bv"], m)
    kIc = csa.csa_compress_packed(d["kI"], pk, d["wi"], d["bi"], m)
    idx = csa.csa_indexer_topk_packed(d["qI"], d["wI"], kIc, pk, m, k)
    out, lse = csa.csa_sparse_mqa_packed(d["q"], pk, csa.KVCache(k=Kc, v=Vc), m, idx, d["K"], d["V"], win,
                                         1 / np.sqrt(192))
    torch.cuda.synchronize()
    sc = 1 / np.sqrt(192)
    for s, n in enumerate(lens):
        t0 = pk.cu_tokens_host[s]
        sl = slice(t0, t0 + n)
        Kc_o = _round_bf16(R.compress(f64(K[sl])[None], f64(wk), f64(bk), m, 2 * m))
        Vc_o = _round_bf16(R.compress(f64(V[sl])[None], f64(wv), f64(bv), m, 2 * m))
        kI_o = _round_bf16(R.compress(f64(kI[sl])[None], f64(wi), f64(bi), m, 2 * m))
        sc_o = R.indexer_scores(f64(qI[sl])[None], f64(wI[sl])[None], kI_o, np.arange(n), m)
        ref_idx = R.topk_set(sc_o, k)
        got_idx = idx[sl].cpu().numpy()[None]
        same = check_topk(got_idx, sc_o, ref_idx, k, f"packed indexer seq {s}")
        use = np.where(same.reshape(1, n)[..., None], ref_idx, got_idx.astype(np.int64))
        O, L = R.csa_sparse_mqa(f64(q[sl])[None], np.arange(n), Kc_o, Vc_o, use, m, f64(K[sl])[None],
                                f64(V[sl])[None], 0, win, sc)
        assert_close(f64(out[sl])[None], O, f"packed attention seq {s}")
        assert_lse(f64(lse[sl])[None], L, f"packed lse seq {s}")


@pytest.mark.parametrize("H", [16, 64])
def test_packed_hca_prefill_is_per_sequence(H):
    g = np.random.default_rng(100 + H)
    mp, win = 128, 128
    lens = [1000, 5, 129, 384, 2000]
    pk = csa.Packed(lens, mp)
    TT = pk.total_tokens
    q, K, V = _bf16(g, (TT, H, 192)), _bf16(g, (TT, 192)), _bf16(g, (TT, 128))
    wk, bk, wv, bv = _f32(g, (192,), 0.02), _f32(g, (mp, 192), 0.1), _f32(g, (128,), 0.02), _f32(g, (mp, 128), 0.1)
    Kc = csa.hca_compress_packed(K.to(DEV), pk, wk.to(DEV), bk.to(DEV), mp)
    Vc = csa.hca_compress_packed(V.to(DEV), pk, wv.to(DEV), bv.to(DEV), mp)
    out, lse = csa.hca_dense_mqa_packed(q.to(DEV), pk, csa.KVCache(k=Kc, v=Vc), mp, K.to(DEV), V.to(DEV), win, 0.08)
    torch.cuda.synchronize()
    for s, n in enumerate(lens):
        t0 = pk.cu_tokens_host[s]
        sl = slice(t0, t0 + n)
        Kc_o = _round_bf16(R.compress(f64(K[sl])[None], f64(wk), f64(bk), mp, mp))
        Vc_o = _round_bf16(R.compress(f64(V[sl])[None], f64(wv), f64(bv), mp, mp))
        O, L = R.hca_dense_mqa(f64(q[sl])[None], np.arange(n), Kc_o, Vc_o, mp, f64(K[sl])[None], f64(V[sl])[None], 0,
                               win, 0.08)
        assert_close(f64(out[sl])[None], O, f"packed hca seq {s}")
        assert_lse(f64(lse[sl])[None], L, f"packed hca lse seq {s}")
