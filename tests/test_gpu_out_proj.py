"""GPU parity of the grouped output projection (csa_grouped_out_proj) against
the float64 oracle: decode-sized and prefill-sized row counts, ragged row
tiles, every tile width the kernel picks (64, 128, 256 channels), one group and
one head per group."""
import numpy as np
import pytest
import torch

import long_context_sparse_10_b200 as csa
from oracle import csa_ref as R
from parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("rows,H,G,dg", [
    (8, 64, 8, 1024),      # 1M-context decode: 8 rows, narrow tiles
    (300, 64, 8, 512),     # ragged row tiles, 128-wide tiles
    (2000, 64, 8, 1024),   # many row tiles: 256-wide tiles, persistent CTAs with several tiles each
    (1000, 16, 1, 256),    # one group: K = 2048
    (129, 16, 16, 64),     # one head per group: K = 128
])
def test_grouped_out_proj(rows, H, G, dg):
    g = np.random.default_rng(rows + H + G + dg)
    o = torch.from_numpy((g.standard_normal((rows, H, 128)) * 0.5).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((g.standard_normal((G, dg, (H // G) * 128)) * 0.02).astype(np.float32)).to(torch.bfloat16)
    y = csa.grouped_out_proj(o.to(DEV), w.to(DEV))
    torch.cuda.synchronize()
    ref = R.grouped_out_proj(f64(o), f64(w))
    assert y.shape == ref.shape
    assert_close(f64(y), ref, f"grouped out proj rows={rows} G={G} dg={dg}")


def test_grouped_out_proj_twice_in_a_row_is_identical():
    g = np.random.default_rng(9)
    o = torch.from_numpy(g.standard_normal((700, 64, 128)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    w = torch.from_numpy((g.standard_normal((8, 1024, 1024)) * 0.02).astype(np.float32)).to(torch.bfloat16).to(DEV)
    a = csa.grouped_out_proj(o, w)
    b = csa.grouped_out_proj(o, w)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
