"""GPU parity of the Mamba-2 path against the fp64 oracle (all calls go through
the C interface of librs_b200.so)."""
import numpy as np
import pytest
import torch

import rs_decode_outputs_b200 as rs
from oracle.replay_model import RingPointers
from tests.harness import (TOL_BF16, TOL_E4M3, TOL_F32, Mamba2Case, check_copy_is_quantised_master,
                           make_session, out_err, rel_err)

pytestmark = pytest.mark.gpu


def decode_run(case, sess, steps, K, check_ptrs=True, check_drift=False, errs=None):
    """Append / decode / commit-at-K loop; returns the max relative error."""
    ptr = RingPointers(case.B, sess.cfg.cap)
    worst = 0.0
    for t in range(steps):
        s = case.draw(1)
        sess.append(s, 1)
        ptr.append(1)
        y = sess.decode()
        ref, _ = case.oracle_run(s)
        e = out_err(case.gpu_pairs(y), ref[0], sess.cfg.copy_dtype)
        worst = max(worst, e)
        if errs is not None:
            errs.append(e)
        if ptr.length[0] >= K:
            sess.commit(min_len=K)
            ptr.commit(min_len=K)
            if check_drift:
                check_copy_is_quantised_master(sess)
        if check_ptrs:
            head, tail = sess.read_ptrs()
            assert np.array_equal(head, ptr.head) and np.array_equal(tail, ptr.tail), t
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()
    return worst


def test_config0_fp32_from_zero(cuda_device):
    """The tiny fp32 case: B=2, H=4, P=N=16, G=1, fp32 throughout, K=4, 32 steps, seed 0."""
    case = Mamba2Case(2, 4, 16, 16, 1, rs.RS_F32, seed=0, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, 2, 4, 16, 16, cap=4, in_dtype=rs.RS_F32,
                        copy_dtype=rs.RS_NONE, A=case.A, D=case.D)
    err = decode_run(case, sess, 32, K=4)
    assert err <= TOL_F32, err
    # the fp32 master after the last commit is the oracle state
    m = sess.master().double().cpu().numpy()
    assert rel_err(m.reshape(2, 4, -1), case.hstate.reshape(2, 4, -1)) <= 1e-5


@pytest.mark.parametrize("copy,tol", [(rs.RS_BF16, TOL_BF16), (rs.RS_E4M3, TOL_E4M3),
                                      (rs.RS_NONE, TOL_F32)])
def test_ragged_shapes_with_copies(cuda_device, copy, tol):
    """Several tiles, rows not a multiple of a pass, 2 groups, ring wrap-around,
    commit interval not dividing the step count; checkpoint from a prefill."""
    B, H, P, N, G, K = 3, 6, 40, 128, 2, 5
    case = Mamba2Case(B, H, P, N, G, rs.RS_BF16, seed=11, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, B, H, P, N, G, cap=8, copy_dtype=copy, A=case.A, D=case.D)
    # prefill 24 steps eagerly in fp32 on the GPU, then load it as the checkpoint
    state = torch.zeros(B, H, P, N, device=cuda_device)
    pre = case.draw(24)
    sess.eager_step(state, rs.RS_F32, pre, 24)
    case.oracle_run(pre)
    sess.load_checkpoint(state)
    if copy != rs.RS_NONE:
        check_copy_is_quantised_master(sess)
    err = decode_run(case, sess, 23, K=K, check_drift=copy != rs.RS_NONE)
    assert err <= tol, err


def test_verify_rollback_spec_rounds(cuda_device):
    """Speculative rounds: append 5, verify 5 outputs in one pass, roll back the
    rejected suffix by pointer, commit at len >= 8.  Outputs at every position
    equal the oracle's eager outputs of that extension of the accepted history."""
    B, H, P, N, G = 4, 3, 32, 64, 1
    case = Mamba2Case(B, H, P, N, G, rs.RS_BF16, seed=21, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, B, H, P, N, G, cap=16, npos_max=5, copy_dtype=rs.RS_BF16,
                        A=case.A, D=case.D)
    acc = rs.inputs.acceptance(12, B, 4, 0.7, seed=5)
    ptr = RingPointers(B, 16)
    worst = 0.0
    for r in range(12):
        s = case.draw(5)
        sess.append(s, 5)
        ptr.append(5)
        y = sess.verify(5)
        ref, _ = case.oracle_run(s, advance=False)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref))
        a = acc[r].numpy()
        k = torch.tensor(4 - a, dtype=torch.int32, device=cuda_device)
        sess.rollback(k)
        ptr.rollback(4 - a)
        # oracle: advance each pair over its 1 + a accepted entries
        x, dt, Bm, C = case.pair_inputs(s)
        for i, (b, h) in enumerate(case.pairs):
            n = 1 + int(a[b])
            import oracle
            _, case.hstate[i] = oracle.mamba2_eager(float(case.A[h]), float(case.D[h]), x[i, :n],
                                                    dt[i, :n], Bm[i, :n], C[i, :n],
                                                    h0=case.hstate[i])
        sess.commit(min_len=8)
        ptr.commit(min_len=8)
        head, tail = sess.read_ptrs()
        assert np.array_equal(head, ptr.head) and np.array_equal(tail, ptr.tail), r
    assert worst <= TOL_BF16, worst
    status, _ = sess.get_error()
    assert status == rs.RS_OK


def test_rollback_then_continue_is_bit_identical_to_truncated_run(cuda_device):
    B, H, P, N = 2, 4, 64, 128
    case = Mamba2Case(B, H, P, N, 1, rs.RS_BF16, seed=31, device=cuda_device)
    s = case.draw(7)
    first = {k: v[:2].contiguous() for k, v in s.items()}
    junk = {k: v[2:5].contiguous() for k, v in s.items()}
    more = {k: v[5:7].contiguous() for k, v in s.items()}
    outs = []
    for variant in ("rollback", "truncated"):
        sess = make_session(rs.RS_MAMBA2, B, H, P, N, cap=8, npos_max=2, A=case.A, D=case.D)
        state = torch.randn(B, H, P, N, device=cuda_device, generator=torch.Generator(
            device=cuda_device).manual_seed(3)) * 0.1
        sess.load_checkpoint(state)
        sess.append(first, 2)
        if variant == "rollback":
            sess.append(junk, 3)
            sess.rollback(torch.full((B,), 3, dtype=torch.int32, device=cuda_device))
        sess.append(more, 2)
        outs.append((sess.decode(), sess.verify(2), sess.read_ptrs()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][2][1], outs[1][2][1])


def test_device_errors_are_sticky_and_leave_pointers(cuda_device):
    B, H, P, N = 3, 2, 16, 32
    case = Mamba2Case(B, H, P, N, 1, rs.RS_BF16, seed=41, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, B, H, P, N, cap=8, npos_max=4, A=case.A, D=case.D)
    y = sess.decode()                               # empty buffer
    assert torch.count_nonzero(y) == 0
    st, flags = sess.get_error()
    assert st == rs.RS_ERR_DEVICE_FLAG and np.all(flags == rs.RS_SEQ_ERR_EMPTY)
    sess.clear_error()
    sess.append(case.draw(5), 5)
    sess.append(case.draw(5), 5)                    # 10 > cap 8: refused
    head, tail = sess.read_ptrs()
    assert np.all(tail == 5) and np.all(head == 0)
    st, flags = sess.get_error()
    assert np.all(flags == rs.RS_SEQ_ERR_OVERFLOW)
    sess.clear_error()
    sess.rollback(torch.tensor([1, 6, -1], dtype=torch.int32, device=cuda_device))
    head, tail = sess.read_ptrs()
    assert list(tail) == [4, 5, 5]
    st, flags = sess.get_error()
    assert list(flags) == [0, rs.RS_SEQ_ERR_ROLLBACK, rs.RS_SEQ_ERR_ROLLBACK]
    sess.clear_error()
    with pytest.raises(rs.RsError):
        sess.verify(5)                              # npos > npos_max: host refuses
    with pytest.raises(rs.RsError):
        sess.append(case.draw(9), 9)                # T > cap: host refuses


@pytest.mark.parametrize("sdt,tol", [(rs.RS_F32, TOL_F32), (rs.RS_BF16, 5e-2)])
def test_eager_baseline_kernel(cuda_device, sdt, tol):
    B, H, P, N, G = 3, 4, 48, 64, 2
    case = Mamba2Case(B, H, P, N, G, rs.RS_BF16, seed=51, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, B, H, P, N, G, cap=8, A=case.A, D=case.D)
    state = torch.zeros(B, H, P, N, device=cuda_device, dtype=torch.float32 if sdt == rs.RS_F32 else torch.bfloat16)
    worst = 0.0
    for t in range(20):
        s = case.draw(1)
        y = sess.eager_step(state, sdt, s, 1)
        ref, _ = case.oracle_run(s)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref))
    s = case.draw(6)                                # several steps in one launch
    y = sess.eager_step(state, sdt, s, 6)
    ref, _ = case.oracle_run(s)
    worst = max(worst, rel_err(case.gpu_pairs(y), ref))
    assert worst <= tol, worst


def test_eager_verify_slots_and_accept(cuda_device):
    B, H, P, N = 2, 3, 32, 64
    case = Mamba2Case(B, H, P, N, 1, rs.RS_BF16, seed=61, device=cuda_device)
    sess = make_session(rs.RS_MAMBA2, B, H, P, N, cap=8, npos_max=4, A=case.A, D=case.D)
    slots = torch.zeros(5, B, H, P, N, device=cuda_device)
    cur = torch.zeros(B, dtype=torch.int32, device=cuda_device)
    acc = rs.inputs.acceptance(6, B, 3, 0.7, seed=9)
    import oracle
    worst = 0.0
    for r in range(6):
        s = case.draw(4)
        y = sess.eager_verify(slots, rs.RS_F32, cur, s, 4)
        ref, _ = case.oracle_run(s, advance=False)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref))
        keep = 1 + acc[r].numpy()
        sess.eager_accept(cur, torch.tensor(keep, dtype=torch.int32, device=cuda_device))
        x, dt, Bm, C = case.pair_inputs(s)
        for i, (b, h) in enumerate(case.pairs):
            n = int(keep[b])
            _, case.hstate[i] = oracle.mamba2_eager(float(case.A[h]), float(case.D[h]), x[i, :n],
                                                    dt[i, :n], Bm[i, :n], C[i, :n],
                                                    h0=case.hstate[i])
    assert worst <= TOL_F32, worst
