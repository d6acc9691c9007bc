"""Property checks of the workspace layout (host code, no GPU) over random
valid configurations: every region is 256-byte aligned, regions do not
overlap and lie inside the reported total, and each region has the size its
layout in include/rs.h states.  Also: the newer entry points refuse NULL
arguments before any CUDA call."""
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import rs_decode_outputs_b200 as rs

REGIONS = ("master", "copy", "scale", "ring_a", "ring_b", "ring_c", "ring_d", "ring_e", "scratch")


def a4(v):
    return (v + 3) // 4 * 4


def expected_scratch_bytes(kind, B, H, G, npos_max, cap, CC):
    npr = 1 if npos_max <= 1 else 2 if npos_max <= 2 else 5 if npos_max <= 5 else 8
    cs = a4(cap) + 4
    tile = a4(16 + npr * cs + (npr * CC if kind == rs.RS_GDN else 0))
    group = a4(npr * CC) if kind == rs.RS_MAMBA2 else 0
    return 4 * (B * H * tile + B * G * group)


@st.composite
def configs(draw):
    kind = draw(st.sampled_from([rs.RS_MAMBA2, rs.RS_GDN]))
    B = draw(st.integers(1, 300))
    G = draw(st.sampled_from([1, 2, 4])) if kind == rs.RS_MAMBA2 else 1
    H = G * draw(st.integers(1, 24))
    R = draw(st.integers(1, 256))
    CC = draw(st.sampled_from([16, 32, 64, 128, 256]))
    cap = draw(st.sampled_from([1, 2, 4, 8, 16, 32, 64, 128, 256]))
    npos_max = draw(st.integers(1, min(8, cap)))
    in_dt = draw(st.sampled_from([rs.RS_F32, rs.RS_BF16]))
    copy = draw(st.sampled_from([rs.RS_NONE, rs.RS_BF16, rs.RS_E4M3]))
    out = draw(st.sampled_from([rs.RS_F32, rs.RS_BF16]))
    shared = draw(st.sampled_from([0, 1])) if copy != rs.RS_NONE else 0
    return rs.make_config(kind, B, H, R, CC, G, cap, npos_max, in_dt, copy, out, shared)


@settings(max_examples=300, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(configs())
def test_layout_regions_are_aligned_disjoint_and_sized(cfg):
    try:
        lay = rs.rs_workspace_layout(cfg)
    except rs.RsError as e:
        assert e.status == rs.RS_ERR_UNSUPPORTED   # register-tile limits only
        return
    B, H, R, CC, G, cap = cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, cfg.ngroups, cfg.cap
    ib = 2 if cfg.in_dtype == rs.RS_BF16 else 4
    E = B * H * R * CC
    capd = max(cap, 4)
    blk_r = (cap * R * ib + 15) // 16 * 16
    blk_c = cap * CC * ib
    assert lay.master_bytes == (0 if cfg.shared_lowp else 4 * E)
    assert lay.copy_bytes == {rs.RS_NONE: 0, rs.RS_BF16: 2 * E, rs.RS_E4M3: E}[cfg.copy_dtype]
    assert lay.scale_bytes == (4 * B * H if cfg.copy_dtype == rs.RS_E4M3 else 0)
    if cfg.kind == rs.RS_MAMBA2:
        sizes = [B * H * blk_r, 4 * B * H * capd, B * G * blk_c, B * G * blk_c, 0]
    else:
        sizes = [B * H * blk_c, B * H * blk_c, B * H * blk_r, 4 * B * H * capd, 4 * B * H * capd]
    assert [getattr(lay, n + "_bytes") for n in ("ring_a", "ring_b", "ring_c", "ring_d", "ring_e")] == sizes
    assert lay.scratch_bytes == expected_scratch_bytes(cfg.kind, B, H, G, cfg.npos_max, cap, CC)
    spans = []
    for n in REGIONS:
        off, size = getattr(lay, n), getattr(lay, n + "_bytes")
        assert off % 256 == 0, n
        if size:
            spans.append((off, off + size, n))
    for n in ("head", "tail", "err", "arrive"):
        off = getattr(lay, n)
        assert off % 256 == 0, n
        spans.append((off, off + 4 * B, n))
    spans.sort()
    for (a0, a1, na), (b0, b1, nb) in zip(spans, spans[1:]):
        assert a1 <= b0, (na, nb)
    assert spans[-1][1] <= lay.total == rs.rs_workspace_size(cfg)


def test_newer_entry_points_refuse_null_arguments():
    lib = rs.library()
    assert lib.rs_decode_step(None, None, 1, None, None) == rs.RS_ERR_ARG
    assert lib.rs_decode_outputs_static_scratch(None, None, None) == rs.RS_ERR_ARG
    assert lib.rs_profile_start(None, 4) == rs.RS_ERR_ARG
    assert lib.rs_profile_stop(None, None, None, None) == rs.RS_ERR_ARG
    assert lib.rs_selftest_bounded_wait(None, 1000, None) == rs.RS_ERR_ARG
