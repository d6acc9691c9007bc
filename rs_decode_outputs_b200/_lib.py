"""ctypes binding of ``librs_b200.so`` (the C interface declared in ``include/rs.h``).

Argument marshalling only: every function here converts torch tensors / Python
values to the C types of the entry point of the same name and raises
``RsError`` on a non-OK status.  Every step of the decode path runs in the CUDA
library; there is no Python or CPU fallback -- importing this module fails
loudly if the library is missing.
"""
import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librs_b200.so")

# enums (values fixed by include/rs.h)
RS_OK, RS_ERR_ARG, RS_ERR_CAPACITY, RS_ERR_CUDA = 0, -1, -2, -4
RS_ERR_WORKSPACE, RS_ERR_DEVICE_FLAG, RS_ERR_UNSUPPORTED = -5, -6, -8
RS_MAMBA2, RS_GDN = 0, 1
RS_NONE, RS_F32, RS_BF16, RS_E4M3 = 0, 1, 2, 3
RS_SEQ_ERR_OVERFLOW, RS_SEQ_ERR_ROLLBACK, RS_SEQ_ERR_EMPTY, RS_SEQ_ERR_TIMEOUT = 1, 2, 4, 8

TORCH_DTYPE = {RS_F32: torch.float32, RS_BF16: torch.bfloat16, RS_E4M3: torch.uint8}


class RsError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = _lib.rs_status_string(status).decode()
        if status == RS_ERR_CUDA:
            msg += ": " + _lib.rs_last_cuda_error().decode()
        super().__init__(f"{where}: {msg} ({status})")


class RsConfig(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("batch", ctypes.c_int32), ("nheads", ctypes.c_int32),
                ("headdim", ctypes.c_int32), ("dstate", ctypes.c_int32),
                ("ngroups", ctypes.c_int32), ("cap", ctypes.c_int32), ("npos_max", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("copy_dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("shared_lowp", ctypes.c_int32),
                ("gdn_scale", ctypes.c_float)]


class RsInputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("x", "dt", "B", "C", "q", "k", "v", "alpha", "beta")]


_sz = ctypes.c_size_t
_LAYOUT_FIELDS = ["master", "master_bytes", "copy", "copy_bytes", "scale", "scale_bytes",
                  "ring_a", "ring_a_bytes", "ring_b", "ring_b_bytes", "ring_c", "ring_c_bytes",
                  "ring_d", "ring_d_bytes", "ring_e", "ring_e_bytes", "head", "tail", "err",
                  "arrive", "scratch", "scratch_bytes", "total"]


class RsLayout(ctypes.Structure):
    _fields_ = [(n, _sz) for n in _LAYOUT_FIELDS]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python rs_decode_outputs_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    P = ctypes.POINTER
    sigs = {
        "rs_workspace_size": [P(RsConfig), P(_sz)],
        "rs_workspace_layout": [P(RsConfig), P(RsLayout)],
        "rs_create": [P(RsConfig), vp, _sz, vp, vp, vp, P(vp)],
        "rs_destroy": [vp],
        "rs_load_checkpoint": [vp, vp, vp],
        "rs_append": [vp, P(RsInputs), i32, vp],
        "rs_decode_outputs": [vp, vp, vp],
        "rs_decode_step": [vp, P(RsInputs), i32, vp, vp],
        "rs_commit": [vp, i32, vp, vp],
        "rs_verify_outputs": [vp, i32, vp, vp],
        "rs_rollback": [vp, vp, vp],
        "rs_eager_step": [vp, vp, i32, P(RsInputs), i32, vp, vp],
        "rs_eager_verify": [vp, vp, i32, vp, P(RsInputs), i32, vp, vp],
        "rs_eager_accept": [vp, vp, vp, vp],
        "rs_get_error": [vp, vp, vp, vp],
        "rs_clear_error": [vp, vp],
        "rs_read_ptrs": [vp, vp, vp, vp],
        "rs_profile_start": [vp, i32],
        "rs_selftest_bounded_wait": [vp, ctypes.c_longlong, vp],
        "rs_decode_outputs_static_scratch": [vp, vp, vp],
        "rs_profile_stop": [vp, vp, vp, vp],
    }
    for name, args in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = st
    lib.rs_status_string.argtypes = [ctypes.c_int]
    lib.rs_status_string.restype = ctypes.c_char_p
    lib.rs_last_cuda_error.argtypes = []
    lib.rs_last_cuda_error.restype = ctypes.c_char_p
    lib.rs_launch_count.argtypes = []
    lib.rs_launch_count.restype = ctypes.c_uint64
    return lib


_lib = _load()


def library():
    return _lib


def _check(status, where):
    if status != RS_OK:
        raise RsError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def make_config(kind, batch, nheads, headdim, dstate, ngroups=1, cap=16, npos_max=1,
                in_dtype=RS_BF16, copy_dtype=RS_BF16, out_dtype=RS_F32, shared_lowp=0,
                gdn_scale=1.0) -> RsConfig:
    return RsConfig(kind, batch, nheads, headdim, dstate, ngroups, cap, npos_max, in_dtype,
                    copy_dtype, out_dtype, shared_lowp, gdn_scale)


def make_inputs(d) -> RsInputs:
    """dict of tensors (keys x, dt, B, C or q, k, v, alpha, beta) -> RsInputs."""
    return RsInputs(*[_ptr(d.get(n)) for n in ("x", "dt", "B", "C", "q", "k", "v", "alpha", "beta")])


def rs_workspace_size(cfg: RsConfig) -> int:
    n = _sz()
    _check(_lib.rs_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "rs_workspace_size")
    return n.value


def rs_workspace_layout(cfg: RsConfig) -> RsLayout:
    lay = RsLayout()
    _check(_lib.rs_workspace_layout(ctypes.byref(cfg), ctypes.byref(lay)), "rs_workspace_layout")
    return lay


def rs_create(cfg, workspace, A, D=None, stream=None):
    h = ctypes.c_void_p()
    _check(_lib.rs_create(ctypes.byref(cfg), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _ptr(A), _ptr(D),
                          _stream(stream), ctypes.byref(h)), "rs_create")
    return h


def rs_destroy(h):
    _check(_lib.rs_destroy(h), "rs_destroy")


def rs_load_checkpoint(h, state, stream=None):
    _check(_lib.rs_load_checkpoint(h, _ptr(state), _stream(stream)), "rs_load_checkpoint")


def rs_append(h, inputs, T, stream=None):
    ins = inputs if isinstance(inputs, RsInputs) else make_inputs(inputs)
    _check(_lib.rs_append(h, ctypes.byref(ins), int(T), _stream(stream)), "rs_append")


def rs_decode_outputs(h, y, stream=None):
    _check(_lib.rs_decode_outputs(h, _ptr(y), _stream(stream)), "rs_decode_outputs")


def rs_decode_outputs_static_scratch(h, y, stream=None):
    _check(_lib.rs_decode_outputs_static_scratch(h, _ptr(y), _stream(stream)),
           "rs_decode_outputs_static_scratch")


def rs_decode_step(h, inputs, T, y, stream=None):
    ins = inputs if isinstance(inputs, RsInputs) else make_inputs(inputs)
    _check(_lib.rs_decode_step(h, ctypes.byref(ins), int(T), _ptr(y), _stream(stream)),
           "rs_decode_step")


def rs_commit(h, min_len=1, mask=None, stream=None):
    _check(_lib.rs_commit(h, int(min_len), _ptr(mask), _stream(stream)), "rs_commit")


def rs_verify_outputs(h, npos, y, stream=None):
    _check(_lib.rs_verify_outputs(h, int(npos), _ptr(y), _stream(stream)), "rs_verify_outputs")


def rs_rollback(h, k, stream=None):
    _check(_lib.rs_rollback(h, _ptr(k), _stream(stream)), "rs_rollback")


def rs_eager_step(h, state, state_dtype, inputs, T, y, stream=None):
    ins = inputs if isinstance(inputs, RsInputs) else make_inputs(inputs)
    _check(_lib.rs_eager_step(h, _ptr(state), int(state_dtype), ctypes.byref(ins), int(T),
                              _ptr(y), _stream(stream)), "rs_eager_step")


def rs_eager_verify(h, slots, state_dtype, cur, inputs, npos, y, stream=None):
    ins = inputs if isinstance(inputs, RsInputs) else make_inputs(inputs)
    _check(_lib.rs_eager_verify(h, _ptr(slots), int(state_dtype), _ptr(cur), ctypes.byref(ins),
                                int(npos), _ptr(y), _stream(stream)), "rs_eager_verify")


def rs_eager_accept(h, cur, keep, stream=None):
    _check(_lib.rs_eager_accept(h, _ptr(cur), _ptr(keep), _stream(stream)), "rs_eager_accept")


def rs_get_error(h, batch, stream=None):
    """Returns (status, per-sequence flags as a numpy uint32 array).  Synchronises."""
    flags = np.zeros(batch, dtype=np.uint32)
    anyv = ctypes.c_uint32()
    s = _lib.rs_get_error(h, flags.ctypes.data, ctypes.byref(anyv), _stream(stream))
    if s not in (RS_OK, RS_ERR_DEVICE_FLAG):
        raise RsError(s, "rs_get_error")
    return s, flags


def rs_clear_error(h, stream=None):
    _check(_lib.rs_clear_error(h, _stream(stream)), "rs_clear_error")


def rs_read_ptrs(h, batch, stream=None):
    head = np.zeros(batch, dtype=np.int32)
    tail = np.zeros(batch, dtype=np.int32)
    _check(_lib.rs_read_ptrs(h, head.ctypes.data, tail.ctypes.data, _stream(stream)),
           "rs_read_ptrs")
    return head, tail


def rs_launch_count() -> int:
    return int(_lib.rs_launch_count())


def rs_profile_start(h, max_calls):
    _check(_lib.rs_profile_start(h, int(max_calls)), "rs_profile_start")


def rs_profile_stop(h):
    """Returns (timed calls, summed prep-kernel ms, summed streaming-kernel ms)."""
    n = ctypes.c_int()
    tp = ctypes.c_float()
    ts = ctypes.c_float()
    _check(_lib.rs_profile_stop(h, ctypes.byref(n), ctypes.byref(tp), ctypes.byref(ts)),
           "rs_profile_stop")
    return n.value, tp.value, ts.value


def rs_selftest_bounded_wait(result, limit_cycles, stream=None):
    _check(_lib.rs_selftest_bounded_wait(_ptr(result), int(limit_cycles), _stream(stream)),
           "rs_selftest_bounded_wait")
