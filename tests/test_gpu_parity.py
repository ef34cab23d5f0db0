"""GPU parity: every C-ABI call against the float64 oracle on the same seeded inputs.

Small and ragged shapes that still span several tiles; edge cases (T < m,
partial tail entries, k > visible entries, exact ties, empty key sets, skipped
index slots, FP8 split cache).  Inputs come from the seeded generator or the
oracle, never from the GPU path.
"""
import math

import numpy as np
import pytest
import torch

import long_context_sparse_10_b200 as csa
from long_context_sparse_10_b200 import synth
from oracle import csa_ref as R
from parity import assert_close, assert_lse, check_topk, e4m3_ordinal, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16(g, shape, std=1.0):
    return torch.from_numpy((g.standard_normal(shape) * std).astype(np.float32)).to(torch.bfloat16)


def _f32(g, shape, std=1.0):
    return torch.from_numpy((g.standard_normal(shape) * std).astype(np.float32))


def _round_bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# compression
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("kind,B,T,d,m", [
    ("csa", 2, 1001, 192, 4), ("csa", 2, 1001, 128, 4), ("csa", 1, 2048, 64, 4), ("csa", 3, 3, 64, 4),
    ("csa", 1, 1, 192, 4), ("csa", 2, 37, 64, 1), ("csa", 1, 130, 256, 16),
    ("hca", 2, 1000, 192, 128), ("hca", 2, 8192, 128, 128), ("hca", 1, 77, 64, 128), ("hca", 1, 300, 64, 33),
])
def test_compress_bf16(kind, B, T, d, m):
    g = np.random.default_rng(11 + T + d)
    cw = 2 * m if kind == "csa" else m
    x = _bf16(g, (B, T, d))
    w = _f32(g, (d,), 0.02 if d != 256 else 0.5)
    b = _f32(g, (cw, d), 0.1 if d != 256 else 2.0)
    fn = csa.csa_compress if kind == "csa" else csa.hca_compress
    y = fn(x.to(DEV), w.to(DEV), b.to(DEV), m)
    torch.cuda.synchronize()
    ref = R.compress(f64(x), f64(w), f64(b), m, cw)
    assert y.shape == ref.shape
    assert_close(f64(y), ref, f"{kind} compress d={d}")


@pytest.mark.parametrize("kind,B,T,m", [("csa", 2, 1001, 4), ("hca", 2, 1000, 128), ("csa", 1, 4096, 4)])
def test_compress_split_fp8(kind, B, T, m):
    g = np.random.default_rng(5 + T)
    cw = 2 * m if kind == "csa" else m
    x = _bf16(g, (B, T, 192))
    w = _f32(g, (192,), 0.02)
    b = _f32(g, (cw, 192), 0.1)
    fn = csa.csa_compress if kind == "csa" else csa.hca_compress
    nope, rope, scale = fn(x.to(DEV), w.to(DEV), b.to(DEV), m, fp8=True)
    torch.cuda.synchronize()
    y = R.compress(f64(x), f64(w), f64(b), m, cw)
    codes, sc = R.quantize_entries(y[..., :128])
    np.testing.assert_allclose(f64(scale), sc, rtol=1e-5)
    d = np.abs(e4m3_ordinal(nope.cpu().numpy()) - e4m3_ordinal(codes))
    assert d.max() <= 1, f"e4m3 codes differ by {d.max()} steps"
    assert (d == 0).mean() > 0.99
    assert_close(f64(rope), y[..., 128:], "rope channels")
    # dequantised nope within half an e4m3 step of the fp64 value (plus the 1-step slack)
    deq = R.e4m3_decode(nope.cpu().numpy()) * f64(scale)[..., None]
    assert np.abs(deq - y[..., :128]).max() <= (32.0 / 448.0) * np.abs(y[..., :128]).max() + 1e-6


# ---------------------------------------------------------------------------
# indexer + top-k
# ---------------------------------------------------------------------------
def _indexer_case(g, B, Tq, N, tie_blocks=0, zero_q=False):
    qI = _bf16(g, (B, Tq, 4, 64))
    if zero_q:
        qI.zero_()
    wI = torch.from_numpy(g.random((B, Tq, 4)).astype(np.float32))
    kI = _bf16(g, (B, N, 64))
    if tie_blocks:
        kI = kI[:, ::tie_blocks].repeat_interleave(tie_blocks, dim=1)[:, :N].contiguous()
    return qI, wI, kI


@pytest.mark.parametrize("B,Tq,N,q_pos0,m,k,ties,zero", [
    (2, 600, 150, 0, 4, 64, 0, False),         # prefill rows (row path), k > visible early on
    (1, 2048, 512, 0, 4, 64, 0, False),        # the T=2048 prefill shape
    (1, 700, 700, 0, 1, 33, 4, False),         # exact ties in blocks of 4
    (1, 400, 100, 0, 4, 16, 0, True),          # all scores zero: lowest indices win
    (3, 1, 50000, 4 * 50000 - 1, 4, 2048, 0, False),  # long rows, all visible
    (2, 1, 50000, 120000 - 1, 4, 64, 0, False),       # long rows, partly visible
    (4, 8, 1000, 3000, 4, 100, 0, False),      # few rows: long-row path with short rows
    (2, 3, 3000, 11999, 4, 2048, 2, False),    # long-row path with ties
    (2, 2, 70, 100, 4, 40, 0, False),          # every row sees fewer than k entries
    (1, 40, 300, 0, 4, 8, 0, False),           # long-row path; the first rows see no entry at all
    (1, 1, 40000, 4 * 40000 - 1, 4, 4096, 0, True),   # long rows, all ties, k = max
    (2, 1, 300001, 4 * 300001 - 1, 4, 2048, 0, False),  # rows past 262144 entries: bitmap in global memory
    (1, 600, 40000, 120000, 4, 512, 0, False),  # more long rows than CTA slots: one chunk per row
    (64, 1, 32768, 4 * 32768 - 1, 4, 2048, 0, False),  # 64 decode rows at 131072 tokens of context
    (2, 1, 2049, 4 * 2049 - 1, 4, 2048, 0, False),    # long rows with one entry more than k visible
    (2, 2, 2048, 4 * 2048 - 2, 4, 2048, 0, False),    # long rows with k - 1 and exactly k entries visible
    (1, 1, 9000, 4 * 9000 - 1, 4, 1003, 8, False),    # long row, a block of 8 exact ties straddling the cut
    # prefill rows at k = 2048 (row path): visible counts crossing k, and near 16384
    (1, 300, 16384, 8000, 4, 2048, 0, False),
    (1, 300, 16384, 65536 - 300, 4, 2048, 0, False),
    # enough prefill rows (>= 32 per SM) for the on-chip tcgen05 kernel
    (3, 1700, 425, 0, 4, 64, 0, False),        # k > visible early on, three sequences
    (1, 5000, 5000, 0, 1, 33, 4, False),       # exact ties in blocks of 4
    (1, 5000, 1250, 0, 4, 16, 0, True),        # all scores zero: lowest indices win
    (1, 4800, 4096, 4000, 4, 2048, 0, False),  # k = 2048, visible counts crossing k
])
def test_indexer_topk(B, Tq, N, q_pos0, m, k, ties, zero):
    g = np.random.default_rng(B * 1000 + N + k)
    qI, wI, kI = _indexer_case(g, B, Tq, N, ties, zero)
    idx = csa.csa_indexer_topk(qI.to(DEV), wI.to(DEV), kI.to(DEV), m, k, q_pos0=q_pos0)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    pos = q_pos0 + np.arange(Tq)
    s = R.indexer_scores(f64(qI), f64(wI), f64(kI), pos, m)
    ref = R.topk_set(s, k)
    same = check_topk(got, s, ref, k, "indexer")
    assert same.mean() > 0.97


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def _oracle_idx(g, B, Tq, N, m, k, q_pos0):
    s = g.standard_normal((B, Tq, N))
    ends = (np.arange(N) + 1) * m - 1
    s = np.where(ends[None, None, :] <= (q_pos0 + np.arange(Tq))[None, :, None], s, -np.inf)
    return R.topk_set(s, k)


@pytest.mark.parametrize("H,B,T,m,k,win,sep_v", [
    (16, 2, 300, 4, 16, 32, True), (64, 1, 200, 4, 64, 128, True), (16, 1, 2048, 4, 64, 128, True),
    (64, 2, 150, 4, 8, 7, False),
    # 64 heads, 5 tiles of 128 slots per late row: the K/V stage rings wrap and their barrier phases flip
    (64, 1, 2000, 4, 512, 128, True),    # separate V: 2 stages
    (64, 1, 2000, 4, 512, 128, False),   # V = K[:, :128]: 3 stages
    # 16 heads, many rows: query-blocked kernel over the union of 16 queries' selections
    (16, 2, 333, 4, 24, 0, False),       # ragged last block, no window, V = K[:, :128]
    (16, 1, 1500, 4, 128, 128, True),    # 16 x 128 selections per block: the largest union
])
def test_csa_sparse_mqa_prefill_bf16(H, B, T, m, k, win, sep_v):
    g = np.random.default_rng(H + T + k)
    N = -(-T // m)
    q = _bf16(g, (B, T, H, 192))
    Kc = _bf16(g, (B, N, 192))
    Vc = _bf16(g, (B, N, 128)) if sep_v else None
    Kr = _bf16(g, (B, T, 192))
    Vr = _bf16(g, (B, T, 128)) if sep_v else None
    idx = _oracle_idx(g, B, T, N, m, k, 0)
    # exercise skipped slots: out of range, future entries
    idx[:, ::7, 0] = N + 5
    idx[:, 1::5, -1] = N - 1
    sc = 1 / math.sqrt(192)
    cache = csa.KVCache(k=Kc.to(DEV), v=None if Vc is None else Vc.to(DEV))
    winw = csa.Window(k=Kr.to(DEV), v=None if Vr is None else Vr.to(DEV), pos0=0, length=win)
    out, lse = csa.csa_sparse_mqa(q.to(DEV), cache, m, torch.from_numpy(idx.astype(np.int32)).to(DEV), winw, sc)
    torch.cuda.synchronize()
    Vc64 = f64(Vc) if Vc is not None else f64(Kc)[..., :128]
    Vr64 = f64(Vr) if Vr is not None else f64(Kr)[..., :128]
    O, L = R.csa_sparse_mqa(f64(q), np.arange(T), f64(Kc), Vc64, idx, m, f64(Kr), Vr64, 0, win, sc)
    assert_close(f64(out), O, f"csa prefill H={H}")
    assert_lse(f64(lse), L, "csa prefill lse")


@pytest.mark.parametrize("H,B,T,mp,win", [
    (16, 2, 700, 32, 64), (64, 1, 1000, 128, 128), (16, 1, 129, 128, 1),
    # more query blocks than SMs (a persistent CTA runs several): no window, so the first block of each
    # sequence sees no key at all; the last block of each sequence holds 8 queries (its second row group
    # lies past the sequence and is zero-filled)
    (16, 3, 1000, 32, 0),
    (16, 2, 2500, 64, 128),  # several blocks per CTA with a window; last block of 4 queries
])
def test_hca_dense_mqa_prefill_bf16(H, B, T, mp, win):
    g = np.random.default_rng(H * T + mp)
    N = -(-T // mp)
    q = _bf16(g, (B, T, H, 192))
    Kc, Vc = _bf16(g, (B, N, 192)), _bf16(g, (B, N, 128))
    Kr, Vr = _bf16(g, (B, T, 192)), _bf16(g, (B, T, 128))
    sc = 0.08
    out, lse = csa.hca_dense_mqa(q.to(DEV), csa.KVCache(k=Kc.to(DEV), v=Vc.to(DEV)), mp,
                                 csa.Window(k=Kr.to(DEV), v=Vr.to(DEV), pos0=0, length=win), sc)
    torch.cuda.synchronize()
    O, L = R.hca_dense_mqa(f64(q), np.arange(T), f64(Kc), f64(Vc), mp, f64(Kr), f64(Vr), 0, win, sc)
    assert_close(f64(out), O, f"hca prefill H={H}")
    assert_lse(f64(lse), L, "hca prefill lse")


def _split_cache(g, B, N):
    x = torch.from_numpy(g.standard_normal((B, N, 192)).astype(np.float32))
    return synth.split_fp8_cache(x)


@pytest.mark.parametrize("kind,H,B,N,k,win,Tq,max_sms", [
    ("csa", 64, 3, 5000, 512, 128, 1, 0), ("csa", 16, 2, 3000, 2048, 128, 1, 0), ("hca", 64, 2, 3000, 0, 128, 1, 0),
    ("hca", 16, 3, 700, 0, 64, 1, 0), ("csa", 64, 2, 4000, 256, 128, 4, 0),
    # rows split over many CTAs whose partial states merge through global records
    ("hca", 64, 8, 8192, 0, 128, 1, 0),   # the 1M-context decode's HCA shape: 17 CTAs per row
    ("hca", 64, 2, 30000, 0, 128, 1, 0),  # 59 CTAs per row, last split ragged
    ("csa", 64, 8, 40000, 2048, 128, 1, 0),  # the 1M-context decode's CSA shape (cluster merge)
    ("hca", 64, 1, 30000, 0, 128, 4, 0),  # several query rows of one sequence, each split over CTAs
    # an SM budget: 10 CTAs of 7 tiles per row (last ragged), 2 CTAs per row, one CTA per row
    ("hca", 64, 8, 8192, 0, 128, 1, 80), ("hca", 64, 8, 8192, 0, 128, 1, 16), ("hca", 64, 8, 8192, 0, 128, 1, 3),
])
def test_decode_split_fp8(kind, H, B, N, k, win, Tq, max_sms):
    g = np.random.default_rng(N + H + k)
    m = 4 if kind == "csa" else 128
    L = N * m
    q_pos0 = L - Tq
    nope, rope, scale = _split_cache(g, B, N)
    q = _bf16(g, (B, Tq, H, 192))
    Wk = _bf16(g, (B, win + Tq, 192))
    wpos0 = L - Tq - win
    cache = csa.KVCache(nope=nope.to(DEV), rope=rope.to(DEV), scale=scale.to(DEV))
    w = csa.Window(k=Wk.to(DEV), pos0=wpos0, length=win)
    sc = 1 / math.sqrt(192)
    K64, V64 = R.dequant_split(nope.numpy(), f64(rope), scale.numpy())
    if kind == "csa":
        idx = _oracle_idx(g, B, Tq, N, m, k, q_pos0)
        out, lse = csa.csa_sparse_mqa(q.to(DEV), cache, m, torch.from_numpy(idx.astype(np.int32)).to(DEV), w, sc,
                                      q_pos0=q_pos0)
        O, Ls = R.csa_sparse_mqa(f64(q), q_pos0 + np.arange(Tq), K64, V64, idx, m, f64(Wk), f64(Wk)[..., :128],
                                 wpos0, win, sc)
    else:
        out, lse = csa.hca_dense_mqa(q.to(DEV), cache, m, w, sc, q_pos0=q_pos0, max_sms=max_sms)
        O, Ls = R.hca_dense_mqa(f64(q), q_pos0 + np.arange(Tq), K64, V64, m, f64(Wk), f64(Wk)[..., :128], wpos0,
                                win, sc)
    torch.cuda.synchronize()
    assert_close(f64(out), O, f"{kind} decode fp8 H={H}")
    assert_lse(f64(lse), Ls, f"{kind} decode lse")


def _exact_split_cache(g, B, N, positive):
    """Split cache whose widened keys are exact in bf16 (E4M3 codes times a power-of-two scale), so that
    logits far from 1 do not magnify the key rounding of the tcgen05 path."""
    codes = g.integers(0, 256, size=(B, N, 128)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] ^= 0x01  # no NaN codes
    if positive:
        codes &= 0x7F
    rope = g.standard_normal((B, N, 64)).astype(np.float32)
    if positive:
        rope = np.abs(rope)
    scale = np.full((B, N), 2.0 ** -7, np.float32)
    return torch.from_numpy(codes), torch.from_numpy(rope).to(torch.bfloat16), torch.from_numpy(scale)


@pytest.mark.parametrize("kind,case", [("csa", "large"), ("hca", "large"), ("csa", "negative"), ("hca", "negative"),
                                       ("csa", "mixed"), ("hca", "mixed"), ("csa", "low"), ("hca", "low")])
def test_decode_logit_ranges(kind, case):
    """Logits outside the first tile's trial reference: above 2^20 for some heads (large), below 2^-64 for every
    head (negative: positive keys, negative queries), or below it for half of the heads only (mixed); and
    logits inside it but far below 0 for every head (low)."""
    g = np.random.default_rng({"large": 1, "negative": 2, "mixed": 3, "low": 4}[case] + (10 if kind == "hca" else 0))
    H, B, N, win = 64, 2, 3000, 128
    m = 4 if kind == "csa" else 128
    k = 512
    L = N * m
    q_pos0 = L - 1
    positive = case != "large"
    nope, rope, scale = _exact_split_cache(g, B, N, positive)
    qf = g.standard_normal((B, 1, H, 192)).astype(np.float32)
    wf = g.standard_normal((B, win + 1, 192)).astype(np.float32)
    sc = 1 / math.sqrt(192)
    if case == "large":
        sc *= 16.0
    elif case in ("negative", "low"):
        wf = np.abs(wf)
        qf = -np.abs(qf) * 2.0
        sc *= 8.0 if case == "negative" else 4.0
    else:
        wf = np.abs(wf)
        qf[:, :, :32] = -np.abs(qf[:, :, :32]) * 16.0
    q = torch.from_numpy(qf).to(torch.bfloat16)
    Wk = torch.from_numpy(wf).to(torch.bfloat16)
    wpos0 = L - 1 - win
    cache = csa.KVCache(nope=nope.to(DEV), rope=rope.to(DEV), scale=scale.to(DEV))
    w = csa.Window(k=Wk.to(DEV), pos0=wpos0, length=win)
    K64, V64 = R.dequant_split(nope.numpy(), f64(rope), scale.numpy())
    if kind == "csa":
        idx = _oracle_idx(g, B, 1, N, m, k, q_pos0)
        out, lse = csa.csa_sparse_mqa(q.to(DEV), cache, m, torch.from_numpy(idx.astype(np.int32)).to(DEV), w, sc,
                                      q_pos0=q_pos0)
        O, Ls = R.csa_sparse_mqa(f64(q), q_pos0 + np.arange(1), K64, V64, idx, m, f64(Wk), f64(Wk)[..., :128],
                                 wpos0, win, sc)
    else:
        out, lse = csa.hca_dense_mqa(q.to(DEV), cache, m, w, sc, q_pos0=q_pos0)
        O, Ls = R.hca_dense_mqa(f64(q), q_pos0 + np.arange(1), K64, V64, m, f64(Wk), f64(Wk)[..., :128], wpos0,
                                win, sc)
    torch.cuda.synchronize()
    assert_close(f64(out), O, f"{kind} decode logits {case}")
    assert_lse(f64(lse), Ls, f"{kind} decode lse, logits {case}")


def test_attention_with_no_keys_outputs_zero():
    g = np.random.default_rng(3)
    B, T, H, m = 1, 8, 16, 4
    q = _bf16(g, (B, T, H, 192))
    Kc = _bf16(g, (B, 2, 192))
    idx = torch.full((B, T, 4), -1, dtype=torch.int32)
    out, lse = csa.csa_sparse_mqa(q.to(DEV), csa.KVCache(k=Kc.to(DEV)), m, idx.to(DEV), None, 0.1)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.cpu()) == 0
    assert torch.isneginf(lse.cpu()).all()


# ---------------------------------------------------------------------------
# whole pipelines at the small workload sizes
# ---------------------------------------------------------------------------
def test_csa_prefill_pipeline_t2048():
    wl = synth.WORKLOADS["csa_prefill_t2048"]
    x = synth.prefill_inputs(wl, seed=0)
    m, k, win, T = wl.m, wl.k, wl.win, wl.T
    sc = 1 / math.sqrt(192)
    d = {kk: v.to(DEV) for kk, v in x.items()}
    Kc = csa.csa_compress(d["k"], d["w_k"], d["b_k"], m)
    Vc = csa.csa_compress(d["v"], d["w_v"], d["b_v"], m)
    kIc = csa.csa_compress(d["kI"], d["w_i"], d["b_i"], m)
    idx = csa.csa_indexer_topk(d["qI"], d["wI"], kIc, m, k)
    out, lse = csa.csa_sparse_mqa(d["q"], csa.KVCache(k=Kc, v=Vc), m, idx,
                                  csa.Window(k=d["k"], v=d["v"], pos0=0, length=win), sc)
    torch.cuda.synchronize()
    # oracle pipeline: compressed entries are stored as bf16 (the cache's storage type)
    Kc_o = f64(_round_bf16(R.compress(f64(x["k"]), f64(x["w_k"]), f64(x["b_k"]), m, 2 * m)))
    Vc_o = f64(_round_bf16(R.compress(f64(x["v"]), f64(x["w_v"]), f64(x["b_v"]), m, 2 * m)))
    kI_o = f64(_round_bf16(R.compress(f64(x["kI"]), f64(x["w_i"]), f64(x["b_i"]), m, 2 * m)))
    assert_close(f64(Kc), Kc_o, "Kc", max_abs=1.6e-2)
    s = R.indexer_scores(f64(x["qI"]), f64(x["wI"]), kI_o, np.arange(T), m)
    ref_idx = R.topk_set(s, k)
    same = check_topk(idx.cpu().numpy(), s, ref_idx, k, "pipeline indexer")
    O, L = R.csa_sparse_mqa(f64(x["q"]), np.arange(T), Kc_o, Vc_o, ref_idx, m, f64(x["k"]), f64(x["v"]), 0, win, sc)
    rows = same.reshape(1, T)
    assert rows.mean() > 0.95
    assert_close(f64(out)[rows], O[rows], "pipeline output")
    assert_lse(f64(lse)[rows], L[rows], "pipeline lse")


def test_hca_prefill_pipeline_t8192():
    wl = synth.WORKLOADS["hca_prefill_t8192"]
    x = synth.prefill_inputs(wl, seed=0)
    mp, win, T = wl.m, wl.win, wl.T
    sc = 1 / math.sqrt(192)
    d = {kk: v.to(DEV) for kk, v in x.items()}
    Kc = csa.hca_compress(d["k"], d["w_k"], d["b_k"], mp)
    Vc = csa.hca_compress(d["v"], d["w_v"], d["b_v"], mp)
    assert Kc.shape[1] == 64
    out, lse = csa.hca_dense_mqa(d["q"], csa.KVCache(k=Kc, v=Vc), mp, csa.Window(k=d["k"], v=d["v"], length=win), sc)
    torch.cuda.synchronize()
    Kc_o = f64(_round_bf16(R.compress(f64(x["k"]), f64(x["w_k"]), f64(x["b_k"]), mp, mp)))
    Vc_o = f64(_round_bf16(R.compress(f64(x["v"]), f64(x["w_v"]), f64(x["b_v"]), mp, mp)))
    assert_close(f64(Kc), Kc_o, "HCA Kc", max_abs=1.6e-2)
    rows = np.arange(0, T, 3)       # every third query row of both sequences
    O, L = R.hca_dense_mqa(f64(x["q"][:, rows]), rows, Kc_o, Vc_o, mp, f64(x["k"]), f64(x["v"]), 0, win, sc)
    assert_close(f64(out[:, rows]), O, "HCA pipeline output")
    assert_lse(f64(lse[:, rows]), L, "HCA pipeline lse")


def test_no_device_timeouts_recorded():
    # every bounded wait in the tensor-core attention kernels completed in the tests above
    from long_context_sparse_10_b200 import _lib
    lib = _lib.load()
    assert lib.csa_check_device_error(torch.cuda.current_stream().cuda_stream) == 0, lib.csa_last_error()


@pytest.mark.parametrize("B,Tq,N,q_pos0,m,k,head_scale", [
    (3, 1, 50000, 4 * 50000 - 1, 4, 2048, None),     # long rows (decode)
    (2, 1, 30000, 100000, 4, 512, None),             # long rows, partly visible
    (1, 600, 150, 0, 4, 64, None),                   # prefill rows
    # query heads far outside fp16's range in both directions (the kernel
    # rescales each head by a power of two before its fp16 MMA)
    (2, 1, 20000, 4 * 20000 - 1, 4, 256, (2.0 ** -40, 2.0 ** 30, 1.0, 2.0 ** -10)),
    (1, 40, 300, 0, 4, 32, (2.0 ** 25, 2.0 ** -35, 0.0, 1.0)),
    (3, 1, 20001, 4 * 20001 - 1, 4, 4096, None),     # odd N, k at its maximum
])
def test_indexer_topk_e4m3_keys(B, Tq, N, q_pos0, m, k, head_scale):
    g = np.random.default_rng(N + k + 17)
    qI = _bf16(g, (B, Tq, 4, 64))
    if head_scale is not None:
        qI = (qI.float() * torch.tensor(head_scale).view(1, 1, 4, 1)).to(torch.bfloat16)
    wI = torch.from_numpy(g.random((B, Tq, 4)).astype(np.float32))
    codes, scale = synth.fp8_rows(torch.from_numpy(g.standard_normal((B, N, 64)).astype(np.float32)))
    idx = csa.csa_indexer_topk_e4m3(qI.to(DEV), wI.to(DEV), codes.to(DEV), scale.to(DEV), m, k, q_pos0=q_pos0)
    torch.cuda.synchronize()
    kI = R.e4m3_decode(codes.numpy()) * scale.double().numpy()[..., None]
    s = R.indexer_scores(f64(qI), f64(wI), kI, q_pos0 + np.arange(Tq), m)
    same = check_topk(idx.cpu().numpy(), s, R.topk_set(s, k), k, "indexer e4m3")
    assert same.mean() > 0.97


def test_empty_calls_return_without_work():
    """No query rows (Tq = 0): the calls return empty outputs and launch nothing."""
    lib = csa._lib.load()
    before = lib.csa_launch_count()
    q = torch.empty(1, 0, 64, 192, dtype=torch.bfloat16, device=DEV)
    nope = torch.zeros(1, 4, 128, dtype=torch.uint8, device=DEV)
    rope = torch.zeros(1, 4, 64, dtype=torch.bfloat16, device=DEV)
    scale = torch.ones(1, 4, dtype=torch.float32, device=DEV)
    out, lse = csa.hca_dense_mqa(q, csa.KVCache(nope=nope, rope=rope, scale=scale), 128, None, 0.1)
    idx = csa.csa_indexer_topk(torch.empty(2, 0, 4, 64, dtype=torch.bfloat16, device=DEV),
                               torch.empty(2, 0, 4, device=DEV), torch.zeros(2, 8, 64, dtype=torch.bfloat16, device=DEV),
                               4, 4)
    torch.cuda.synchronize()
    assert out.numel() == 0 and lse.numel() == 0 and idx.shape == (2, 0, 4)
    assert lib.csa_launch_count() == before


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_decode_split_fp8_separate_window_values(kind):
    """FP8 cache with a raw window that carries its own values (the warp-MMA kernel's case)."""
    g = np.random.default_rng(41)
    H, B, N, win = 64, 2, 2000, 128
    m = 4 if kind == "csa" else 128
    k = 256
    L = N * m
    q_pos0 = L - 1
    nope, rope, scale = _split_cache(g, B, N)
    q = _bf16(g, (B, 1, H, 192))
    Wk = _bf16(g, (B, win + 1, 192))
    Wv = _bf16(g, (B, win + 1, 128))
    wpos0 = L - 1 - win
    cache = csa.KVCache(nope=nope.to(DEV), rope=rope.to(DEV), scale=scale.to(DEV))
    w = csa.Window(k=Wk.to(DEV), v=Wv.to(DEV), pos0=wpos0, length=win)
    sc = 1 / math.sqrt(192)
    K64, V64 = R.dequant_split(nope.numpy(), f64(rope), scale.numpy())
    if kind == "csa":
        idx = _oracle_idx(g, B, 1, N, m, k, q_pos0)
        out, lse = csa.csa_sparse_mqa(q.to(DEV), cache, m, torch.from_numpy(idx.astype(np.int32)).to(DEV), w, sc,
                                      q_pos0=q_pos0)
        O, Ls = R.csa_sparse_mqa(f64(q), q_pos0 + np.arange(1), K64, V64, idx, m, f64(Wk), f64(Wv), wpos0, win, sc)
    else:
        out, lse = csa.hca_dense_mqa(q.to(DEV), cache, m, w, sc, q_pos0=q_pos0)
        O, Ls = R.hca_dense_mqa(f64(q), q_pos0 + np.arange(1), K64, V64, m, f64(Wk), f64(Wv), wpos0, win, sc)
    torch.cuda.synchronize()
    assert_close(f64(out), O, f"{kind} decode fp8, separate window V")
    assert_lse(f64(lse), Ls, f"{kind} decode lse, separate window V")


def test_csa_prefill_pipeline_t65536_sampled_rows():
    """The 65,536-token CSA prefill (64 heads, k = 2048, separate V) through the whole GPU pipeline, at full
    size, checked on sampled query rows: rows that see fewer than k entries, rows around the point where
    selection becomes partial (t = 8191), and a stride over the rest (up to 17 key tiles per row)."""
    wl = synth.WORKLOADS["csa_prefill_t65536"]
    x = synth.prefill_inputs(wl, seed=0)
    m, k, win, T = wl.m, wl.k, wl.win, wl.T
    sc = 1 / math.sqrt(192)
    d = {kk: v.to(DEV) for kk, v in x.items()}
    Kc = csa.csa_compress(d["k"], d["w_k"], d["b_k"], m)
    Vc = csa.csa_compress(d["v"], d["w_v"], d["b_v"], m)
    kIc = csa.csa_compress(d["kI"], d["w_i"], d["b_i"], m)
    idx = csa.csa_indexer_topk(d["qI"], d["wI"], kIc, m, k)
    out, lse = csa.csa_sparse_mqa(d["q"], csa.KVCache(k=Kc, v=Vc), m, idx,
                                  csa.Window(k=d["k"], v=d["v"], pos0=0, length=win), sc)
    torch.cuda.synchronize()
    Kc_o = f64(_round_bf16(R.compress(f64(x["k"]), f64(x["w_k"]), f64(x["b_k"]), m, 2 * m)))
    Vc_o = f64(_round_bf16(R.compress(f64(x["v"]), f64(x["w_v"]), f64(x["b_v"]), m, 2 * m)))
    kI_o = f64(_round_bf16(R.compress(f64(x["kI"]), f64(x["w_i"]), f64(x["b_i"]), m, 2 * m)))
    assert_close(f64(Kc), Kc_o, "Kc", max_abs=1.6e-2)
    assert_close(f64(Vc), Vc_o, "Vc", max_abs=1.6e-2)
    assert_close(f64(kIc), kI_o, "kIc", max_abs=1.6e-2)
    g = np.random.default_rng(65536)
    rows = np.unique(np.concatenate([
        np.arange(0, 130, 7),                                   # window still filling, few entries
        g.choice(np.arange(130, 8100), 60, replace=False),      # every visible entry selected
        np.arange(8180, 8200),                                  # selection turns partial at t = 8191
        g.choice(np.arange(8200, T), 200, replace=False), [T - 1]]))
    s = R.indexer_scores(f64(x["qI"][:, rows]), f64(x["wI"][:, rows]), kI_o, rows, m)
    ref_idx = R.topk_set(s, k)
    got_idx = idx[:, rows].cpu().numpy()
    same = check_topk(got_idx, s, ref_idx, k, "t65536 indexer")
    assert same.mean() > 0.9
    use = np.where(same.reshape(1, -1)[..., None], ref_idx, got_idx.astype(np.int64))
    O, L = R.csa_sparse_mqa(f64(x["q"][:, rows]), rows, Kc_o, Vc_o, use, m, f64(x["k"]), f64(x["v"]), 0, win, sc)
    assert_close(f64(out[:, rows]), O, "t65536 attention")
    assert_lse(f64(lse[:, rows]), L, "t65536 lse")


@pytest.mark.parametrize("B,Tq,N,q_pos0,m,k,head_scale", [
    (3, 1, 50000, 4 * 50000 - 1, 4, 2048, None),     # long rows (decode)
    (2, 1, 30000, 100000, 4, 512, None),             # long rows, partly visible
    (1, 600, 150, 0, 4, 64, None),                   # prefill rows (row path)
    (2, 1, 20000, 4 * 20000 - 1, 4, 256, (2.0 ** -40, 2.0 ** 30, 1.0, 2.0 ** -10)),
    (1, 300, 4000, 16000 - 300, 4, 2048, None),      # prefill rows at k = 2048
    (8, 1, 262144, 4 * 262144 - 1, 4, 2048, None),   # the 1M-context decode shape
])
def test_indexer_topk_e2m1_keys(B, Tq, N, q_pos0, m, k, head_scale):
    """FP4 (E2M1, two codes per byte, per-entry scale) indexer keys: scores of the decoded keys."""
    g = np.random.default_rng(N + k + 29)
    qI = _bf16(g, (B, Tq, 4, 64))
    if head_scale is not None:
        qI = (qI.float() * torch.tensor(head_scale).view(1, 1, 4, 1)).to(torch.bfloat16)
    wI = torch.from_numpy(g.random((B, Tq, 4)).astype(np.float32))
    codes, scale = synth.fp4_rows(torch.from_numpy(g.standard_normal((B, N, 64)).astype(np.float32)))
    assert codes.shape == (B, N, 32)
    idx = csa.csa_indexer_topk_e2m1(qI.to(DEV), wI.to(DEV), codes.to(DEV), scale.to(DEV), m, k, q_pos0=q_pos0)
    torch.cuda.synchronize()
    kI = R.e2m1_unpack(codes.numpy()) * scale.double().numpy()[..., None]
    s = R.indexer_scores(f64(qI), f64(wI), kI, q_pos0 + np.arange(Tq), m)
    same = check_topk(idx.cpu().numpy(), s, R.topk_set(s, k), k, "indexer e2m1")
    assert same.mean() > 0.9
