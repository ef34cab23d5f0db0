"""Failure detection without a GPU fault: a bounded device wait that runs out is
reported by csa_check_device_error as CSA_ERR_DEVICE_TIMEOUT, the record is
cleared by that report, and the context stays usable afterwards.  The wait is
the one every library kernel uses on its barriers, made to run out on a
barrier nothing arrives at (no copy, MMA or TMEM allocation is involved)."""
import numpy as np
import pytest
import torch

import long_context_sparse_10_b200 as csa
from long_context_sparse_10_b200 import _lib

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_once_and_the_context_stays_usable():
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.csa_check_device_error(stream) == _lib.CSA_OK, lib.csa_last_error()
    assert lib.csa_debug_expire_wait(stream) == _lib.CSA_OK, lib.csa_last_error()
    assert lib.csa_check_device_error(stream) == _lib.CSA_ERR_DEVICE_TIMEOUT
    assert b"gave up" in lib.csa_last_error()
    assert lib.csa_check_device_error(stream) == _lib.CSA_OK  # reported once, then cleared
    # a normal call afterwards still computes the right answer
    g = np.random.default_rng(5)
    qI = torch.from_numpy(g.standard_normal((1, 1, 4, 64)).astype(np.float32)).to(torch.bfloat16).cuda()
    wI = torch.ones(1, 1, 4, device="cuda")
    kI = torch.zeros(1, 64, 64, dtype=torch.bfloat16, device="cuda")
    kI[0, 37] = qI[0, 0, 0]  # the only entry with a positive score
    idx = csa.csa_indexer_topk(qI, wI, kI, 4, 1, q_pos0=4 * 64 - 1)
    torch.cuda.synchronize()
    assert int(idx[0, 0, 0]) == 37
    assert lib.csa_check_device_error(stream) == _lib.CSA_OK
