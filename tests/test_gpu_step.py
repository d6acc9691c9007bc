"""The fused decode step (rs_decode_step: append + output-only replay in two
kernels) against the composed calls rs_append + rs_decode_outputs /
rs_verify_outputs, and against the fp64 oracle."""
import numpy as np
import pytest
import torch

import rs_decode_outputs_b200 as rs
from oracle.replay_model import RingPointers
from tests.harness import TOL_BF16, TOL_E4M3, GdnCase, Mamba2Case, make_session, out_err

pytestmark = pytest.mark.gpu


def pair(kind, cuda_device, copy=rs.RS_BF16, npos_max=1, cap=8):
    if kind == "m2":
        B, H, R, CC, G = 3, 6, 40, 64, 2
        mk = lambda: Mamba2Case(B, H, R, CC, G, rs.RS_BF16, seed=71, device=cuda_device)
        c0 = mk()
        sessions = [make_session(rs.RS_MAMBA2, B, H, R, CC, G, cap=cap, npos_max=npos_max, copy_dtype=copy,
                                 A=c0.A, D=c0.D) for _ in range(2)]
    else:
        B, H, R, CC = 3, 5, 72, 64
        mk = lambda: GdnCase(B, H, CC, R, rs.RS_BF16, seed=72, device=cuda_device)
        c0 = mk()
        sessions = [make_session(rs.RS_GDN, B, H, R, CC, cap=cap, npos_max=npos_max, copy_dtype=copy)
                    for _ in range(2)]
    return c0, sessions


@pytest.mark.parametrize("kind", ["m2", "gdn"])
@pytest.mark.parametrize("copy", [rs.RS_BF16, rs.RS_E4M3])
def test_step_is_bit_identical_to_append_then_decode(cuda_device, kind, copy):
    case, (fused, composed) = pair(kind, cuda_device, copy)
    ptr = RingPointers(case.B, 8)
    worst = 0.0
    for t in range(21):
        s = case.draw(1)
        y1 = fused.decode_step(s, 1)
        composed.append(s, 1)
        y2 = composed.decode()
        ptr.append(1)
        assert torch.equal(y1, y2), t
        ref, _ = case.oracle_run(s)
        worst = max(worst, out_err(case.gpu_pairs(y1), ref[0], copy))
        if ptr.length[0] >= 5:
            fused.commit(5)
            composed.commit(5)
            ptr.commit(5)
        for sess in (fused, composed):
            head, tail = sess.read_ptrs()
            assert np.array_equal(head, ptr.head) and np.array_equal(tail, ptr.tail), t
    assert torch.equal(fused.workspace, composed.workspace)   # rings, checkpoints, pointers
    assert worst <= (TOL_BF16 if copy == rs.RS_BF16 else TOL_E4M3), worst
    for sess in (fused, composed):
        assert sess.get_error()[0] == rs.RS_OK


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_step_verify_round_matches_append_then_verify(cuda_device, kind):
    case, (fused, composed) = pair(kind, cuda_device, npos_max=5, cap=16)
    for r in range(6):
        s = case.draw(5)
        y1 = fused.decode_step(s, 5)
        composed.append(s, 5)
        y2 = composed.verify(5)
        assert torch.equal(y1, y2), r
        k = torch.full((case.B,), 3, dtype=torch.int32, device=cuda_device)
        fused.rollback(k)
        composed.rollback(k)
        fused.commit(8)
        composed.commit(8)
    assert torch.equal(fused.workspace, composed.workspace)


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_step_overflow_leaves_sequence_unchanged(cuda_device, kind):
    case, (sess, _) = pair(kind, cuda_device, npos_max=2, cap=4)
    sess.decode_step(case.draw(2), 2)
    sess.decode_step(case.draw(2), 2)
    before = sess.workspace.clone()
    y = sess.decode_step(case.draw(2), 2)          # 6 > cap 4: refused on the device
    st, flags = sess.get_error()
    assert st == rs.RS_ERR_DEVICE_FLAG and np.all(flags == rs.RS_SEQ_ERR_OVERFLOW)
    assert torch.count_nonzero(y) == 0
    head, tail = sess.read_ptrs()
    assert np.all(tail == 4) and np.all(head == 0)
    lay = sess.layout
    # everything but the error words and the scratch records is unchanged
    keep = torch.ones_like(before, dtype=torch.bool)
    keep[lay.err:lay.err + 4 * case.B] = False
    keep[lay.scratch:lay.scratch + lay.scratch_bytes] = False
    assert torch.equal(sess.workspace[keep], before[keep])
