"""Edge shapes: the largest state tiles the register-tile kernels take, a
single sequence with a single head, a verify call with exactly npos buffered
entries, and a shape too large for the streaming kernel's stage ring, which
rs_create refuses before launching anything."""
import numpy as np
import pytest
import torch

import rs_decode_outputs_b200 as rs
from tests.harness import TOL_BF16, TOL_F32, GdnCase, Mamba2Case, make_session, rel_err

pytestmark = pytest.mark.gpu


def run_decode(case, sess, steps, K, tol):
    worst = 0.0
    for t in range(steps):
        s = case.draw(1)
        y = sess.decode_step(s, 1)
        ref, _ = case.oracle_run(s)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref[0]))
        if (t + 1) % K == 0:
            sess.commit(K)
    assert worst <= tol, worst
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()


@pytest.mark.parametrize("R,CC", [(256, 64), (64, 256)])
def test_largest_mamba2_tiles(cuda_device, R, CC):
    """The register-tile limits of the state-rewriting kernels: 256 rows with
    64 columns, or 64 rows with 256 columns (four 128-byte boxes per row)."""
    case = Mamba2Case(3, 2, R, CC, 1, rs.RS_BF16, seed=401, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, 3, 2, R, CC, cap=4, A=case.A.to(cuda_device), D=case.D.to(cuda_device))
    run_decode(case, sess, 10, 4, TOL_BF16)


def test_largest_gdn_tile(cuda_device):
    """dv = 256 rows x dk = 64 columns."""
    case = GdnCase(2, 3, 64, 256, rs.RS_BF16, seed=402, device=cuda_device)
    sess = make_session(rs.RS_GDN, 2, 3, 256, 64, cap=4)
    run_decode(case, sess, 10, 4, TOL_BF16)


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_single_sequence_single_head(cuda_device, kind):
    if kind == "m2":
        case = Mamba2Case(1, 1, 16, 16, 1, rs.RS_F32, seed=403, device=cuda_device)
        sess = make_session(rs.RS_MAMBA2, 1, 1, 16, 16, cap=2, in_dtype=rs.RS_F32, copy_dtype=rs.RS_NONE,
                            A=case.A.to(cuda_device), D=case.D.to(cuda_device))
    else:
        case = GdnCase(1, 1, 16, 16, rs.RS_F32, seed=404, device=cuda_device)
        sess = make_session(rs.RS_GDN, 1, 1, 16, 16, cap=2, in_dtype=rs.RS_F32, copy_dtype=rs.RS_NONE)
    run_decode(case, sess, 9, 2, TOL_F32)


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_verify_with_exactly_npos_entries(cuda_device, kind):
    """npos = npos_max = cap = 4: the whole ring is the verified window."""
    if kind == "m2":
        case = Mamba2Case(2, 3, 32, 32, 1, rs.RS_BF16, seed=405, device=cuda_device)
        sess = make_session(rs.RS_MAMBA2, 2, 3, 32, 32, cap=4, npos_max=4, A=case.A.to(cuda_device),
                            D=case.D.to(cuda_device))
    else:
        case = GdnCase(2, 3, 32, 32, rs.RS_BF16, seed=406, device=cuda_device)
        sess = make_session(rs.RS_GDN, 2, 3, 32, 32, cap=4, npos_max=4)
    s = case.draw(4)
    y = sess.decode_step(s, 4)
    ref, _ = case.oracle_run(s)
    assert rel_err(case.gpu_pairs(y), ref) <= TOL_BF16
    head, tail = sess.read_ptrs()
    assert np.all(tail - head == 4)
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()


def test_shape_too_large_for_the_stage_ring_is_refused(cuda_device):
    # 256 x 64 tiles with a ring of 256 slots: each tile's ring block is 128 KB,
    # so three stages of the streaming kernel's ring cannot fit in shared memory
    cfg = rs.make_config(rs.RS_MAMBA2, 2, 2, 256, 64, 1, cap=256)
    ws = torch.zeros(rs.rs_workspace_size(cfg), dtype=torch.uint8, device=cuda_device)
    A = -torch.ones(2, device=cuda_device)
    with pytest.raises(rs.RsError) as ei:
        rs.rs_create(cfg, ws, A)
    assert ei.value.status == rs.RS_ERR_UNSUPPORTED
