"""Context-parallel decode on one GPU: the G ranks' steps run one after another
with the library's kernels (local indexer top-k with scores, candidate merge,
partial attentions, partial merge), the exchange being the concatenation that
an all-gather produces.  The merged result must equal the float64 oracle run
on the whole sequence (selection: exact outside the tie band; attention:
max-abs 2e-2, rel-L2 5e-3; lse within 4e-3)."""
import math

import numpy as np
import pytest
import torch

import long_context_sparse_10_b200 as csa
from long_context_sparse_10_b200 import context_parallel as cp
from long_context_sparse_10_b200 import synth
from oracle import csa_ref as R
from parity import assert_close, assert_lse, check_topk, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _split(nope, rope, scale, lo, hi):
    return csa.KVCache(nope=nope[:, lo:hi].contiguous(), rope=rope[:, lo:hi].contiguous(),
                       scale=scale[:, lo:hi].contiguous())


@pytest.mark.parametrize("world,B,N,k", [(2, 2, 40000, 2048), (3, 1, 30001, 512), (8, 2, 262144, 2048)])
def test_cp_csa_and_hca_decode_match_the_whole_sequence(world, B, N, k):
    g = np.random.default_rng(world * 1000 + N)
    m, mh, win, H = 4, 128, 128, 64
    L = N * m
    t = L - 1
    NH = L // mh
    sc = 1 / math.sqrt(192)
    qI = torch.from_numpy(g.standard_normal((B, 1, 4, 64)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    wI = torch.from_numpy(g.random((B, 1, 4)).astype(np.float32)).to(DEV)
    kI = torch.from_numpy(g.standard_normal((B, N, 64)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    nope, rope, scale = synth.split_fp8_cache(torch.from_numpy(g.standard_normal((B, N, 192)).astype(np.float32)))
    hn, hr, hs = synth.split_fp8_cache(torch.from_numpy(g.standard_normal((B, NH, 192)).astype(np.float32)))
    q = torch.from_numpy(g.standard_normal((B, 1, H, 192)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    hq = torch.from_numpy(g.standard_normal((B, 1, H, 192)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    wk = torch.from_numpy(g.standard_normal((B, win, 192)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    W = csa.Window(k=wk, pos0=L - win, length=win)
    nope, rope, scale, hn, hr, hs = (x.to(DEV) for x in (nope, rope, scale, hn, hr, hs))
    ops = cp.KernelOps()
    shards = [cp.shard_range(N, world, r) for r in range(world)]
    hshards = [cp.shard_range(NH, world, r) for r in range(world)]
    # phase 1 on every rank, "all-gather" = the list in rank order, merge
    cands = [cp.local_candidates(ops, sh, qI, wI, kI[:, sh.lo:sh.hi].contiguous(), m, k, t) for sh in shards]
    sel = cp.merge_candidates(ops, [c[0] for c in cands], [c[1] for c in cands], k)
    parts = [cp.local_sparse_attention(ops, sh, q, _split(nope, rope, scale, sh.lo, sh.hi), m, sel, W, sc, t)
             for sh in shards]
    out, lse = ops.attn_merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    hparts = [cp.local_dense_attention(ops, sh, hq, _split(hn, hr, hs, sh.lo, sh.hi), mh, W, sc, t) for sh in hshards]
    hout, hlse = ops.attn_merge(torch.stack([p[0] for p in hparts]), torch.stack([p[1] for p in hparts]))
    torch.cuda.synchronize()
    # the oracle on the whole sequence
    s = R.indexer_scores(f64(qI), f64(wI), f64(kI), np.array([t]), m)
    ref_sel = R.topk_set(s, k)
    got_sel = sel.cpu().numpy()
    same = check_topk(got_sel, s, ref_sel, k, f"cp{world} selection")
    use = np.where(same.reshape(B, 1)[..., None], ref_sel, got_sel.astype(np.int64))
    K64, V64 = R.dequant_split(nope.cpu().numpy(), f64(rope), scale.cpu().numpy())
    O, Lo = R.csa_sparse_mqa(f64(q), np.array([t]), K64, V64, use, m, f64(wk), f64(wk)[..., :128], L - win, win, sc)
    assert_close(f64(out), O, f"cp{world} csa attention")
    assert_lse(f64(lse), Lo, f"cp{world} csa lse")
    HK, HV = R.dequant_split(hn.cpu().numpy(), f64(hr), hs.cpu().numpy())
    HO, HL = R.hca_dense_mqa(f64(hq), np.array([t]), HK, HV, mh, f64(wk), f64(wk)[..., :128], L - win, win, sc)
    assert_close(f64(hout), HO, f"cp{world} hca attention")
    assert_lse(f64(hlse), HL, f"cp{world} hca lse")


def test_cp_topk_merge_ties_and_padding():
    """Merged candidates: ties go to the lower index across ranks; fewer valid candidates than k pad with -1."""
    ops = cp.KernelOps()
    cs = torch.tensor([[[5.0, 3.0, -np.inf], [5.0, 3.0, 9.0]]], device=DEV).reshape(1, 1, 6)
    ci = torch.tensor([[[2, 7, -1], [11, 12, 30]]], dtype=torch.int32, device=DEV).reshape(1, 1, 6)
    assert ops.topk_merge(cs, ci, 2).cpu().tolist() == [[[2, 30]]]          # 9 and the first 5
    assert ops.topk_merge(cs, ci, 3).cpu().tolist() == [[[2, 11, 30]]]
    assert ops.topk_merge(cs, ci, 7).cpu().tolist() == [[[2, 7, 11, 12, 30, -1, -1]]]
