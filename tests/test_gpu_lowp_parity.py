"""The low-precision arms against the oracle replaying from the same
quantised checkpoint.

A kernel that reads the bf16 or E4M3 copy cannot be closer to the fp64 truth
than the copy's own rounding allows; the sharp check is therefore against the
oracle fed the dequantised checkpoint (oracle state -> fp32 -> the copy's
format -> fp64), which isolates the kernels' own arithmetic.  The two
quantisations see fp32 masters that differ by fp32 rounding (GPU) versus fp64
(oracle), so a code can round the other way now and then; one such flip moves
a (sequence, head) output by well under 1e-2 of its norm, hence the bound.

Both arms are covered: the dual-precision arm (fp32 master + copy) and the
shared low-precision arm, whose commit folds the buffer into the dequantised
copy and quantises again.  Against the fp64 truth the dual arm must meet the
copy-format tolerance on the measure the harness's out_err defines."""
import pytest
import torch

import rs_decode_outputs_b200 as rs
from tests.harness import (TOL_BF16, TOL_E4M3, GdnCase, Mamba2Case, QuantCheckpoint, make_session,
                           out_err, rel_err)

pytestmark = pytest.mark.gpu

TOL_QUANT_ORACLE = 1e-2


def build(kind, copy, shared, cuda_device, npos_max=1, cap=8):
    if kind == "m2":
        B, H, P, N, G = 3, 4, 48, 64, 2
        case = Mamba2Case(B, H, P, N, G, rs.RS_BF16, seed=201, device=cuda_device)
        sess = make_session(rs.RS_MAMBA2, B, H, P, N, G, cap=cap, npos_max=npos_max, copy_dtype=copy,
                            shared_lowp=shared, A=case.A.to(cuda_device), D=case.D.to(cuda_device))
    else:
        B, H, dk, dv = 3, 4, 64, 40
        case = GdnCase(B, H, dk, dv, rs.RS_BF16, seed=202, device=cuda_device, scale=0.125)
        sess = make_session(rs.RS_GDN, B, H, dv, dk, cap=cap, npos_max=npos_max, copy_dtype=copy,
                            shared_lowp=shared, gdn_scale=0.125)
    return case, sess


@pytest.mark.parametrize("kind", ["m2", "gdn"])
@pytest.mark.parametrize("copy", [rs.RS_BF16, rs.RS_E4M3])
@pytest.mark.parametrize("shared", [0, 1])
def test_decode_matches_oracle_on_quantised_checkpoint(cuda_device, kind, copy, shared):
    case, sess = build(kind, copy, shared, cuda_device)
    trk = QuantCheckpoint(case, copy, shared)
    K, steps = 4, 48
    worst_q, truth = 0.0, []
    for t in range(steps):
        s = case.draw(1)
        y = sess.decode_step(s, 1)
        ref_q = trk.step(s)
        ref, _ = case.oracle_run(s)
        got = case.gpu_pairs(y)
        worst_q = max(worst_q, rel_err(got, ref_q[0]))
        truth.append(out_err(got, ref[0], copy))
        if (t + 1) % K == 0:
            sess.commit(K)
            trk.commit()
    assert worst_q <= TOL_QUANT_ORACLE, worst_q
    if not shared:
        tol = TOL_BF16 if copy == rs.RS_BF16 else TOL_E4M3
        assert max(truth) <= tol, max(truth)
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()


@pytest.mark.parametrize("kind", ["m2", "gdn"])
@pytest.mark.parametrize("shared", [0, 1])
def test_verify_matches_oracle_on_quantised_checkpoint(cuda_device, kind, shared):
    """Multi-position verification of 4 drafted positions from the E4M3 copy,
    with the 4th position rejected (rollback by 1) every round."""
    copy = rs.RS_E4M3
    case, sess = build(kind, copy, shared, cuda_device, npos_max=4, cap=16)
    trk = QuantCheckpoint(case, copy, shared)
    worst_q = 0.0
    for r in range(10):
        s = case.draw(4)
        y = sess.decode_step(s, 4)
        keep = {k: v[:3] for k, v in s.items()}
        ref_q = trk.step(s)
        worst_q = max(worst_q, rel_err(case.gpu_pairs(y), ref_q))
        # the oracle takes the accepted prefix only
        trk.buf[-1] = keep
        case.oracle_run(keep)
        sess.rollback(torch.full((case.B,), 1, dtype=torch.int32, device=cuda_device))
        if r % 2 == 1:
            sess.commit(6)
            trk.commit()
    assert worst_q <= TOL_QUANT_ORACLE, worst_q
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()
