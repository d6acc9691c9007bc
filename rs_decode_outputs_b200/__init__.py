"""ReplaySSM decode for Mamba-2 and Gated DeltaNet layers on B200 (sm_100a).

The compute lives in ``librs_b200.so`` (hand-written CUDA behind the C
interface of ``include/rs.h``); this package is its ctypes binding
(``_lib``), a workspace-owning convenience wrapper (``session``) and the
seeded synthetic input generators (``inputs``).
"""
from ._lib import (  # noqa: F401
    RS_BF16, RS_E4M3, RS_ERR_ARG, RS_ERR_CAPACITY, RS_ERR_CUDA, RS_ERR_DEVICE_FLAG,
    RS_ERR_UNSUPPORTED, RS_ERR_WORKSPACE, RS_F32, RS_GDN, RS_MAMBA2, RS_NONE, RS_OK,
    RS_SEQ_ERR_EMPTY, RS_SEQ_ERR_OVERFLOW, RS_SEQ_ERR_ROLLBACK, RS_SEQ_ERR_TIMEOUT, RsConfig,
    RsError, RsInputs, RsLayout, library, make_config, make_inputs, rs_append, rs_clear_error,
    rs_commit, rs_create, rs_decode_outputs, rs_decode_outputs_static_scratch, rs_decode_step, rs_destroy, rs_eager_accept, rs_eager_step,
    rs_eager_verify, rs_get_error, rs_launch_count, rs_load_checkpoint, rs_profile_start, rs_profile_stop, rs_read_ptrs, rs_selftest_bounded_wait,
    rs_rollback, rs_verify_outputs, rs_workspace_layout, rs_workspace_size)
from .session import ReplaySSM  # noqa: F401
