"""Speculative verification across ring-row widths.  The tensor-core path of
the streaming kernel sums the buffer terms as extra MMA k-steps over the
tile's ring block (bf16 rows, rings of up to 32 slots, rows a multiple of 8
elements) and per lane otherwise; these shapes cover rows of 16 to 256
elements, rings of 2 to 32 slots, rows that are a multiple of 8 but not of
16 elements, and a row width that takes the per-lane sum.  Each round
appends npos entries, verifies all npos outputs against the fp64 oracle,
rolls back a Bernoulli suffix and commits the long sequences, so the ring
wraps many times.  The GDN prep takes its Gram form for bf16 inputs and rings
of up to 32 slots and the sequential sweep otherwise (a 64-slot ring, fp32
inputs): both are covered, the fp32 ones at the fp32 tolerance."""
import numpy as np
import pytest
import torch

import oracle
import rs_decode_outputs_b200 as rs
from tests.harness import TOL_BF16, TOL_F32, GdnCase, Mamba2Case, f64, make_session, rel_err

pytestmark = pytest.mark.gpu

B, H = 3, 4

SHAPES = [
    # kind, R, CC, G, cap, npos
    ("m2", 16, 64, 2, 8, 5),     # one 16-row block, two groups
    ("m2", 32, 32, 1, 32, 8),    # 32 slots, 8 positions
    ("m2", 48, 64, 1, 16, 5),
    ("m2", 40, 32, 1, 8, 4),     # rows a multiple of 8, not of 16: last block clamped
    ("m2", 64, 128, 1, 2, 2),    # 2 slots
    ("m2", 256, 64, 1, 8, 5),    # 16 row blocks
    ("m2", 64, 64, 1, 64, 5),    # 64 slots: buffer terms summed per lane
    ("gdn", 128, 64, 1, 32, 5),  # 32 slots
    ("gdn", 32, 128, 1, 4, 3),   # 4 slots
    ("gdn", 24, 64, 1, 16, 5),
    ("gdn", 64, 64, 1, 64, 5),   # 64 slots: sequential sweep in the prep
    # stages of about 68 KB (a 32 KB tile and a 32 KB ring block): three consumer teams instead of four
    ("gdn", 256, 64, 1, 64, 5),
    ("m2", 256, 64, 1, 64, 5),
]
# fp32 inputs, fp32 checkpoint without a copy (CUDA-core contraction, sequential sweep)
SHAPES_F32 = [("m2", 32, 64, 2, 8, 5), ("gdn", 32, 64, 1, 8, 5), ("gdn", 48, 32, 1, 16, 8)]


def setup(kind, R, CC, G, cap, npos, dev, seed, in_dtype=rs.RS_BF16, copy=rs.RS_BF16, scale=1.0):
    if kind == "m2":
        case = Mamba2Case(B, H, R, CC, G, in_dtype, seed, dev)
        sess = make_session(rs.RS_MAMBA2, B, H, R, CC, G, cap=cap, npos_max=npos, in_dtype=in_dtype, copy_dtype=copy,
                            A=case.A, D=case.D)
    else:
        case = GdnCase(B, H, CC, R, in_dtype, seed, dev, scale=scale)
        sess = make_session(rs.RS_GDN, B, H, R, CC, cap=cap, npos_max=npos, in_dtype=in_dtype, copy_dtype=copy,
                            gdn_scale=scale)
    g = torch.Generator(device=dev).manual_seed(seed)
    state = 0.2 * torch.randn(B, H, R, CC, device=dev, generator=g)
    sess.load_checkpoint(state)
    case.hstate = f64(state)[case.pb, case.ph].copy()
    return case, sess


def advance(case, kind, s, keep):
    """Oracle state of every pair after its accepted prefix of s."""
    if kind == "m2":
        x, dt, Bm, C = case.pair_inputs(s)
        A, D = f64(case.A)[case.ph], f64(case.D)[case.ph]
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


@pytest.mark.parametrize("kind,R,CC,G,cap,npos", SHAPES,
                         ids=[f"{k}-R{r}-C{c}-cap{cp}-n{n}" for k, r, c, _, cp, n in SHAPES])
def test_verify_rounds_across_ring_widths(cuda_device, kind, R, CC, G, cap, npos):
    # GDN with an output scale other than 1, so that coef and mul carry it
    case, sess = setup(kind, R, CC, G, cap, npos, cuda_device, seed=700 + R + cap, scale=0.75)
    verify_rounds(case, sess, kind, cap, npos, R, cuda_device, TOL_BF16)


@pytest.mark.parametrize("kind,R,CC,G,cap,npos", SHAPES_F32,
                         ids=[f"{k}-R{r}-C{c}-cap{cp}-n{n}" for k, r, c, _, cp, n in SHAPES_F32])
def test_verify_rounds_fp32(cuda_device, kind, R, CC, G, cap, npos):
    case, sess = setup(kind, R, CC, G, cap, npos, cuda_device, seed=900 + R + cap, in_dtype=rs.RS_F32,
                       copy=rs.RS_NONE)
    verify_rounds(case, sess, kind, cap, npos, R, cuda_device, TOL_F32)


def verify_rounds(case, sess, kind, cap, npos, R, cuda_device, tol):
    rounds = 10
    acc = rs.inputs.acceptance(rounds, B, npos - 1, 0.6, seed=R + cap)
    min_len = cap - npos + 1   # after a commit every length is below this, so npos more entries fit
    length = np.zeros(B, np.int64)
    worst = 0.0
    for r in range(rounds):
        s = case.draw(npos)
        y = sess.decode_step(s, npos)
        ref, _ = case.oracle_run(s, advance=False)
        worst = max(worst, rel_err(case.gpu_pairs(y), ref))
        a = acc[r].numpy()
        sess.rollback(torch.tensor(npos - 1 - a, dtype=torch.int32, device=cuda_device))
        advance(case, kind, s, 1 + a)
        length += 1 + a
        sess.commit(min_len=min_len)
        length[length >= min_len] = 0
        head, tail = sess.read_ptrs()
        assert np.array_equal(tail - head, length), r
    assert worst <= tol, worst
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()
