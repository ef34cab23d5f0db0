"""Context-parallel decode, host logic on CPU ranks (gloo, world size 2 and 3).

Each rank holds a contiguous range of the compressed entries; the ranks
exchange top-k candidates and partial attentions with all_gather.  The compute
steps are replaced here by float64 stand-ins built from the oracle (test
infrastructure; the library runs them as CUDA kernels), so this checks the
orchestration -- ranges, position shifts, index offsets, window ownership and
exchange order -- against the oracle run on the whole sequence by one rank."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_sparse_10_b200 import context_parallel as cp
from oracle import csa_ref as R

B, H, N, M, K, WIN, NH, MH = 2, 4, 300, 4, 24, 16, 40, 32   # N entries (CSA, m=4), NH entries (HCA, m'=32)
L = N * M                                                   # context length; the query sits at t = L - 1


def _inputs():
    g = np.random.default_rng(77)
    d = dict(q=g.standard_normal((B, 1, H, 192)), qI=g.standard_normal((B, 1, 4, 64)), wI=g.random((B, 1, 4)),
             kI=g.standard_normal((B, N, 64)), K=g.standard_normal((B, N, 192)), win=g.standard_normal((B, WIN, 192)),
             hq=g.standard_normal((B, 1, H, 192)), HK=g.standard_normal((B, NH, 192)))
    d["kI"][:, 50:60] = d["kI"][:, 40:50]                   # exact score ties across a shard boundary
    return {k: torch.from_numpy(v) for k, v in d.items()}


class Win:
    def __init__(self, k, pos0, length):
        self.k, self.pos0, self.length = k, pos0, length


class OracleOps:
    """float64 stand-ins for the library calls (same signatures and conventions)."""

    def local_topk(self, qI, wI, kI, m, k, q_pos0):
        s = R.indexer_scores(qI.numpy(), wI.numpy(), kI.numpy(), np.array([q_pos0]), m)
        idx = R.topk_set(s, k)
        sc = np.where(idx >= 0, np.take_along_axis(s, np.maximum(idx, 0), axis=-1), -np.inf)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(sc)

    def topk_merge(self, cs, ci, k):
        cs, ci = cs.numpy(), ci.numpy()
        out = np.full(cs.shape[:-1] + (k,), -1, np.int32)
        for r in np.ndindex(cs.shape[:-1]):
            ok = ci[r] >= 0
            order = np.lexsort((ci[r][ok], -cs[r][ok]))[:k]
            chosen = np.sort(ci[r][ok][order])
            out[r][:len(chosen)] = chosen
        return torch.from_numpy(out)

    def sparse_mqa(self, q, cache, m, idx, win, scale, q_pos0):
        Kc = cache.numpy()
        wk = win.k.numpy() if win is not None else np.zeros((q.shape[0], 0, 192))
        o, lse = R.csa_sparse_mqa(q.numpy(), np.array([q_pos0]), Kc, Kc[..., :128], idx.numpy().astype(np.int64), m,
                                  wk, wk[..., :128], win.pos0 if win else 0, win.length if win else 0,
                                  1 / math.sqrt(192))
        return torch.from_numpy(o), torch.from_numpy(lse)

    def dense_mqa(self, q, cache, m_prime, win, scale, q_pos0):
        Kc = cache.numpy()
        wk = win.k.numpy() if win is not None else np.zeros((q.shape[0], 0, 192))
        o, lse = R.hca_dense_mqa(q.numpy(), np.array([q_pos0]), Kc, Kc[..., :128], m_prime, wk, wk[..., :128],
                                 win.pos0 if win else 0, win.length if win else 0, 1 / math.sqrt(192))
        return torch.from_numpy(o), torch.from_numpy(lse)

    def attn_merge(self, outs, lses):
        o, l = outs.numpy(), lses.numpy()
        mx = l.max(axis=0)
        base = np.where(np.isfinite(mx), mx, 0.0)
        w = np.where(np.isfinite(l), np.exp(l - base), 0.0)
        ws = w.sum(axis=0)
        out = (w[..., None] * o).sum(axis=0) / np.where(ws > 0, ws, 1.0)[..., None]
        lse = np.where(ws > 0, base + np.log(np.where(ws > 0, ws, 1.0)), -np.inf)
        return torch.from_numpy(out), torch.from_numpy(lse)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, ops, t = _inputs(), OracleOps(), L - 1
        sh = cp.shard_range(N, world, rank)
        win = Win(x["win"], L - WIN, WIN)
        out, lse, sel = cp.csa_decode_step(ops, sh, x["q"], x["qI"], x["wI"], x["kI"][:, sh.lo:sh.hi],
                                           x["K"][:, sh.lo:sh.hi], M, K, win, 0.0, t)
        hsh = cp.shard_range(NH, world, rank)
        hout, hlse = cp.hca_decode_step(ops, hsh, x["hq"], x["HK"][:, hsh.lo:hsh.hi], MH, win, 0.0, t)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), out=out.numpy(), lse=lse.numpy(), sel=sel.numpy(),
                 hout=hout.numpy(), hlse=hlse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_equals_single_rank_oracle(tmp_path, world):
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    x = {k: v.numpy() for k, v in _inputs().items()}
    t = L - 1
    s = R.indexer_scores(x["qI"], x["wI"], x["kI"], np.array([t]), M)
    ref_sel = R.topk_set(s, K)
    sc = 1 / math.sqrt(192)
    O, LSE = R.csa_sparse_mqa(x["q"], np.array([t]), x["K"], x["K"][..., :128], ref_sel, M, x["win"],
                              x["win"][..., :128], L - WIN, WIN, sc)
    th = t
    HO, HL = R.hca_dense_mqa(x["hq"], np.array([th]), x["HK"], x["HK"][..., :128], MH, x["win"], x["win"][..., :128],
                             L - WIN, WIN, sc)
    for r in range(world):                      # every rank ends with the whole result
        got = np.load(tmp_path / f"r{r}.npz")
        assert np.array_equal(got["sel"], ref_sel)
        np.testing.assert_allclose(got["out"], O, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(got["lse"], LSE, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got["hout"], HO, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(got["hlse"], HL, rtol=1e-12, atol=1e-12)


def test_shard_ranges_cover_the_entries_in_order():
    for n, w in [(10, 3), (262144, 8), (5, 8), (0, 2)]:
        parts = [cp.shard_range(n, w, r) for r in range(w)]
        assert parts[0].lo == 0 and parts[-1].hi == n
        assert all(a.hi == b.lo for a, b in zip(parts, parts[1:]))
        assert max(p.n for p in parts) - min(p.n for p in parts) <= 1
