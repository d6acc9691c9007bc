"""Host-side checks that need no GPU: the C library loads and exports every
entry point its header declares, the workspace layout is consistent, and bad
configurations / workspaces are refused before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rs.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rs_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def rs():
    from rs_decode_outputs_b200 import build
    build.build()
    import rs_decode_outputs_b200 as rs
    return rs


def test_library_exports_every_declared_symbol(rs):
    names = declared_functions()
    assert len(names) >= 18
    lib = ctypes.CDLL(rs._lib.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    for must in ("rs_create", "rs_append", "rs_decode_outputs", "rs_commit",
                 "rs_verify_outputs", "rs_rollback", "rs_eager_step"):
        assert must in names


def cfg_of(rs, **kw):
    base = dict(kind=rs.RS_MAMBA2, batch=256, nheads=80, headdim=64, dstate=128, ngroups=1,
                cap=16, npos_max=1, in_dtype=rs.RS_BF16, copy_dtype=rs.RS_BF16,
                out_dtype=rs.RS_F32)
    base.update(kw)
    return rs.make_config(**base)


def test_layout_serving_mamba2(rs):
    c = cfg_of(rs)
    lay = rs.rs_workspace_layout(c)
    E = 256 * 80 * 64 * 128
    assert lay.master_bytes == 4 * E and lay.copy_bytes == 2 * E and lay.scale_bytes == 0
    assert lay.ring_a_bytes == 256 * 16 * 80 * 64 * 2          # x
    assert lay.ring_b_bytes == 4 * 256 * 16 * 80                # dt
    assert lay.ring_c_bytes == lay.ring_d_bytes == 256 * 16 * 128 * 2   # B, C (1 group)
    regions = []
    for n in ("master", "copy", "scale", "ring_a", "ring_b", "ring_c", "ring_d", "ring_e"):
        off, sz = getattr(lay, n), getattr(lay, n + "_bytes")
        assert off % 256 == 0
        if sz:
            regions.append((off, off + sz))
    for n in ("head", "tail", "err", "arrive"):
        regions.append((getattr(lay, n), getattr(lay, n) + 4 * 256))
    regions.sort()
    for (a0, a1), (b0, b1) in zip(regions, regions[1:]):
        assert a1 <= b0
    assert regions[-1][1] <= lay.total == rs.rs_workspace_size(c)


def test_layout_gdn_fp8_and_shared(rs):
    c = cfg_of(rs, kind=rs.RS_GDN, nheads=32, headdim=128, dstate=128, cap=32,
               copy_dtype=rs.RS_E4M3)
    lay = rs.rs_workspace_layout(c)
    E = 256 * 32 * 128 * 128
    assert lay.master_bytes == 4 * E and lay.copy_bytes == E and lay.scale_bytes == 4 * 256 * 32
    assert lay.ring_a_bytes == lay.ring_b_bytes == 256 * 32 * 32 * 128 * 2
    assert lay.ring_d_bytes == lay.ring_e_bytes == 4 * 256 * 32 * 32
    shared = rs.rs_workspace_layout(cfg_of(rs, kind=rs.RS_GDN, nheads=32, headdim=128,
                                           dstate=128, cap=32, copy_dtype=rs.RS_E4M3,
                                           shared_lowp=1))
    assert shared.master_bytes == 0 and shared.copy_bytes == E


@pytest.mark.parametrize("bad", [
    dict(kind=7), dict(batch=0), dict(dstate=48), dict(cap=12), dict(cap=512),
    dict(npos_max=9), dict(npos_max=0), dict(in_dtype=3), dict(copy_dtype=1),
    dict(out_dtype=3), dict(shared_lowp=1, copy_dtype=0), dict(ngroups=3),
    dict(kind=1, ngroups=2), dict(headdim=0), dict(headdim=300), dict(gdn_scale=-1.0),
])
def test_bad_configs_are_refused(rs, bad):
    with pytest.raises(rs.RsError) as ei:
        rs.rs_workspace_size(cfg_of(rs, **bad))
    assert ei.value.status == rs.RS_ERR_ARG


def test_too_large_tile_is_unsupported(rs):
    with pytest.raises(rs.RsError) as ei:
        rs.rs_workspace_size(cfg_of(rs, headdim=256, dstate=256))
    assert ei.value.status == rs.RS_ERR_UNSUPPORTED


def test_create_refuses_bad_workspace_before_any_cuda_call(rs):
    lib = rs.library()
    c = cfg_of(rs, batch=2, nheads=4, headdim=16, dstate=16)
    need = rs.rs_workspace_size(c)
    h = ctypes.c_void_p()
    fake_A = ctypes.c_void_p(4096)
    # NULL workspace, misaligned workspace, too small a workspace
    for ws, nbytes in ((None, need), (4096 + 8, need), (4096, need - 1)):
        s = lib.rs_create(ctypes.byref(c), ws, nbytes, fake_A, None, None, ctypes.byref(h))
        assert s == rs.RS_ERR_WORKSPACE and not h.value
    # Mamba-2 needs A
    s = lib.rs_create(ctypes.byref(c), 4096, need, None, None, None, ctypes.byref(h))
    assert s == rs.RS_ERR_ARG


def test_null_handles_and_arguments(rs):
    lib = rs.library()
    assert lib.rs_decode_outputs(None, None, None) == rs.RS_ERR_ARG
    assert lib.rs_commit(None, 1, None, None) == rs.RS_ERR_ARG
    assert lib.rs_rollback(None, None, None) == rs.RS_ERR_ARG
    assert lib.rs_get_error(None, None, None, None) == rs.RS_ERR_ARG
    assert lib.rs_status_string(rs.RS_ERR_CAPACITY) == b"exceeds ring capacity"
    assert rs.rs_launch_count() == 0
