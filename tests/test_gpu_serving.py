"""Parity at the serving shapes (batch 256), in the bench's launch
configuration, on sampled (sequence, head) pairs that the fp64 oracle follows
one by one: the first and last sequences and heads and a spread in between.

  Mamba-2 decode   H=80 P=64 N=128, bf16 inputs, fp32 master + bf16 copy, K=8
  GDN decode       H=32 dk=dv=128, same precisions, K=8
  speculative      rounds on both shapes: 5 positions verified per round,
                   Bernoulli(0.7) acceptance, rollback of the rejected suffix,
                   commit once len >= 16, ring of 32
  E4M3 layers      the hybrid stack's layer shapes (Mamba-2 H=128, GDN H=32)
                   with an E4M3 copy and K=16, dual-precision and
                   shared-low-precision arms

Each starts from a 512-step eager fp32 prefill loaded as the checkpoint (the
oracle runs its own fp64 prefill on the same inputs)."""
import numpy as np
import pytest
import torch

import oracle
import rs_decode_outputs_b200 as rs
from rs_decode_outputs_b200 import inputs as gen
from tests.harness import (TOL_BF16, TOL_E4M3, GdnCase, Mamba2Case, QuantCheckpoint, make_session, out_err,
                           rel_err)

pytestmark = pytest.mark.gpu

BATCH = 256
PREFILL = 512


def sample_pairs(H):
    seqs = [0, 1, 37, 101, 128, 199, 254, 255]
    heads = [0, H - 1, H // 2, 7, H // 3, H - 2, 3, H // 2 + 1]
    return list(zip(seqs, heads)) + [(s, (h + H // 4) % H) for s, h in zip(seqs, heads)]


def m2_setup(dev, H, copy, cap, npos_max=1, shared=0, seed=1):
    case = Mamba2Case(BATCH, H, 64, 128, 1, rs.RS_BF16, seed, dev, pairs=sample_pairs(H), gen_device=dev)
    sess = make_session(rs.RS_MAMBA2, BATCH, H, 64, 128, 1, cap=cap, npos_max=npos_max, copy_dtype=copy,
                        out_dtype=rs.RS_BF16, shared_lowp=shared, A=case.A, D=case.D)
    state = torch.zeros(BATCH, H, 64, 128, device=dev)
    return case, sess, state


def gdn_setup(dev, copy, cap, npos_max=1, shared=0, seed=2, H=32):
    case = GdnCase(BATCH, H, 128, 128, rs.RS_BF16, seed, dev, pairs=sample_pairs(H), gen_device=dev)
    sess = make_session(rs.RS_GDN, BATCH, H, 128, 128, cap=cap, npos_max=npos_max, copy_dtype=copy,
                        out_dtype=rs.RS_BF16, shared_lowp=shared)
    state = torch.zeros(BATCH, H, 128, 128, device=dev)
    return case, sess, state


def prefill(case, sess, state):
    for _ in range(PREFILL // 64):
        s = case.draw(64)
        sess.eager_step(state, rs.RS_F32, s, 64)
        case.oracle_run(s)
    sess.load_checkpoint(state)


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_decode_at_serving_shape(cuda_device, kind):
    case, sess, state = (m2_setup(cuda_device, 80, rs.RS_BF16, 8) if kind == "m2"
                         else gdn_setup(cuda_device, rs.RS_BF16, 8))
    prefill(case, sess, state)
    del state
    worst, K = 0.0, 8
    for t in range(24):
        s = case.draw(1)
        y = sess.decode_step(s, 1)
        ref, _ = case.oracle_run(s)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref[0]))
        if (t + 1) % K == 0:
            sess.commit(K)
    assert worst <= TOL_BF16, worst
    head, tail = sess.read_ptrs()
    assert np.all(head == 24) and np.all(tail == 24)
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()


def advance_pairs(case, kind, s, keep):
    """Oracle state of each sampled pair after its accepted prefix of s."""
    if kind == "m2":
        x, dt, Bm, C = case.pair_inputs(s)
        A = gen_np(case.A)[case.ph]
        D = gen_np(case.D)[case.ph]
        for i, b in enumerate(case.pb):
            n = int(keep[b])
            _, case.hstate[i] = oracle.mamba2_eager(A[i], D[i], x[i, :n], dt[i, :n], Bm[i, :n], C[i, :n],
                                                    h0=case.hstate[i])
    else:
        q, k, v, a, be = case.pair_inputs(s)
        for i, b in enumerate(case.pb):
            n = int(keep[b])
            _, case.hstate[i] = oracle.gdn_eager(q[i, :n], k[i, :n], v[i, :n], a[i, :n], be[i, :n],
                                                 S0=case.hstate[i], scale=case.scale)


def gen_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_speculative_rounds_at_serving_shape(cuda_device, kind):
    npos, cap = 5, 32
    case, sess, state = (m2_setup(cuda_device, 80, rs.RS_BF16, cap, npos_max=npos, seed=3) if kind == "m2"
                         else gdn_setup(cuda_device, rs.RS_BF16, cap, npos_max=npos, seed=3))
    prefill(case, sess, state)
    del state
    acc = gen.acceptance(12, BATCH, npos - 1, 0.7, seed=3)
    length = np.zeros(BATCH, np.int64)
    worst = 0.0
    for r in range(12):
        s = case.draw(npos)
        y = sess.decode_step(s, npos)
        ref, _ = case.oracle_run(s, advance=False)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref))
        a = acc[r].numpy()
        sess.rollback(torch.tensor(npos - 1 - a, dtype=torch.int32, device=cuda_device))
        advance_pairs(case, kind, s, 1 + a)
        length += 1 + a
        sess.commit(min_len=16)
        length[length >= 16] = 0
        head, tail = sess.read_ptrs()
        assert np.array_equal(tail - head, length), r
    assert worst <= TOL_BF16, worst
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_fp8_copy_layer_shapes_dual_and_shared(cuda_device, kind):
    """The hybrid stack's E4M3 layer shapes: errors of both arms at decode steps 1 and 64 on
    the sampled pairs; each arm matches the oracle fed its own quantised
    checkpoint, and the dual arm meets the E4M3 tolerance."""
    K, cap, steps = 16, 16, 64
    errs = {}
    for shared in (0, 1):
        case, sess, state = (m2_setup(cuda_device, 128, rs.RS_E4M3, cap, shared=shared, seed=4000)
                             if kind == "m2" else gdn_setup(cuda_device, rs.RS_E4M3, cap, shared=shared, seed=4008))
        prefill(case, sess, state)
        del state
        trk = QuantCheckpoint(case, rs.RS_E4M3, shared)
        at = {}
        worst_q = 0.0
        for t in range(steps):
            s = case.draw(1)
            y = sess.decode_step(s, 1)
            ref_q = trk.step(s)
            ref, _ = case.oracle_run(s)
            got = case.gpu_pairs(y)
            worst_q = max(worst_q, rel_err(got, ref_q[0]))
            if t + 1 in (1, steps):
                at[t + 1] = out_err(got, ref[0], rs.RS_E4M3)
            if (t + 1) % K == 0:
                sess.commit(K)
                trk.commit()
        assert worst_q <= 1e-2, (shared, worst_q)
        errs[shared] = at
        status, flags = sess.get_error()
        assert status == rs.RS_OK and not flags.any()
        del sess
        torch.cuda.empty_cache()
    assert max(errs[0].values()) <= TOL_E4M3, errs
