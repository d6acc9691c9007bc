"""rs_decode_outputs_static_scratch (replay records in a fixed library-owned
device array) against rs_decode_outputs (records in the workspace scratch):
bit-identical outputs on two consecutive calls, for both layer kinds, and a
handle whose records do not fit the array is refused.  Kept in the last
collected file; it must also pass alone in a fresh process."""
import pytest
import torch

import rs_decode_outputs_b200 as rs
from tests.harness import GdnCase, Mamba2Case, make_session

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["m2", "gdn"])
def test_static_scratch_outputs_equal_workspace_scratch(cuda_device, kind):
    if kind == "m2":
        case = Mamba2Case(3, 6, 40, 64, 2, rs.RS_BF16, seed=301, device=cuda_device)
        sess = make_session(rs.RS_MAMBA2, 3, 6, 40, 64, 2, cap=8, A=case.A.to(cuda_device),
                            D=case.D.to(cuda_device))
    else:
        case = GdnCase(3, 5, 64, 72, rs.RS_BF16, seed=302, device=cuda_device)
        sess = make_session(rs.RS_GDN, 3, 5, 72, 64, cap=8)
    for _ in range(3):
        sess.append(case.draw(1), 1)
    for call in range(2):   # two consecutive calls, a new entry appended in between
        y_ws = sess.decode()
        y_st = sess.new_out()
        rs.rs_decode_outputs_static_scratch(sess.handle, y_st)
        torch.cuda.synchronize()
        assert torch.equal(y_ws, y_st), call
        assert bool(torch.isfinite(y_st.float()).all())
        sess.append(case.draw(1), 1)
    status, flags = sess.get_error()
    assert status == rs.RS_OK and not flags.any()


def test_static_scratch_refuses_records_larger_than_the_array(cuda_device):
    # records of 128 x 128 heads x (16 + 256) floats exceed the 16 MiB array
    sess = make_session(rs.RS_MAMBA2, 128, 128, 16, 16, cap=256,
                        A=-torch.ones(128, device=cuda_device))
    assert sess.layout.scratch_bytes > 16 << 20
    y = sess.new_out()
    with pytest.raises(rs.RsError) as ei:
        rs.rs_decode_outputs_static_scratch(sess.handle, y)
    assert ei.value.status == rs.RS_ERR_CAPACITY
