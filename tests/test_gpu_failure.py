"""Failure detection without a GPU fault: an on-device wait on a barrier that
nothing completes gives up after its bound, reports RS_SEQ_ERR_TIMEOUT, and
the context keeps working (a decode afterwards is checked against the
oracle)."""
import numpy as np
import pytest
import torch

import rs_decode_outputs_b200 as rs
from tests.harness import TOL_F32, Mamba2Case, make_session, rel_err

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable(cuda_device):
    out = torch.zeros(3, dtype=torch.int32, device=cuda_device)
    limit = 2_000_000   # about a millisecond
    rs.rs_selftest_bounded_wait(out, limit)
    got = out.cpu().numpy().astype(np.uint32)
    assert got[0] == rs.RS_SEQ_ERR_TIMEOUT
    waited = int(got[1]) | (int(got[2]) << 32)
    assert waited > limit
    # the library still computes correctly afterwards
    case = Mamba2Case(2, 4, 16, 16, 1, rs.RS_F32, seed=5, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, 2, 4, 16, 16, cap=4, in_dtype=rs.RS_F32, copy_dtype=rs.RS_NONE,
                        A=case.A.to(cuda_device), D=case.D.to(cuda_device))
    worst = 0.0
    for t in range(6):
        s = case.draw(1)
        y = sess.decode_step(s, 1)
        ref, _ = case.oracle_run(s)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref[0]))
        if (t + 1) % 3 == 0:
            sess.commit(3)
    assert worst <= TOL_F32, worst


def test_bounded_wait_rejects_bad_arguments(cuda_device):
    out = torch.zeros(3, dtype=torch.int32, device=cuda_device)
    for limit in (0, 3_000_000_000):
        with pytest.raises(rs.RsError):
            rs.rs_selftest_bounded_wait(out, limit)
