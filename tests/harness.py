"""Helpers shared by the GPU parity tests: run a workload through the CUDA
library and the same inputs through the fp64 oracle, then compare.

Error measure of the tolerances (the pages give "max relative error" and no
norm): for each (sequence, head) output vector of R elements,
||y_gpu - y_oracle||_inf / ||y_oracle||_inf, maximised over vectors and steps
(rel_err).  The E4M3 copy is checked on a whole step's outputs in the same
norm (rel_err_step): its 3 mantissa bits alone can move a single vector by
more than the 6e-2 tolerance, whatever the kernels do, while the step-level
ratio stays near the format's unit roundoff.  The low-precision kernels'
own arithmetic is checked per vector against the oracle fed the same
quantised checkpoint (QuantCheckpoint).
"""
import numpy as np
import torch

import oracle
import rs_decode_outputs_b200 as rs
from rs_decode_outputs_b200 import inputs as gen

TOL_F32 = 1e-4    # fp32 checkpoint / outputs read the fp32 master
TOL_BF16 = 2e-2   # bf16 output copy
TOL_E4M3 = 6e-2   # fp8 E4M3 output copy with a per-(sequence, head) scale

PARAM_SEED_OFFSET = 0
STREAM_SEED_OFFSET = 10_000


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(y, ref):
    """The tolerances' error measure: max over the leading dims (sequence, head,
    position) of ||y - ref||_inf / ||ref||_inf along the last axis, i.e. each
    (sequence, head)'s output vector on its own."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.max(np.abs(y - ref), axis=-1)
    den = np.maximum(np.max(np.abs(ref), axis=-1), 1e-300)
    return float(np.max(num / den))


def rel_err_2(y, ref):
    """max over leading dims of ||y - ref||_2 / ||ref||_2 along the last axis."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.sqrt(np.sum((y - ref) ** 2, axis=-1))
    den = np.maximum(np.sqrt(np.sum(ref ** 2, axis=-1)), 1e-300)
    return float(np.max(num / den))


def rel_err_step(y, ref):
    """||y - ref||_inf / ||ref||_inf over a whole step's outputs (all sequences,
    heads and positions together)."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def out_err(y, ref, copy_dtype):
    """The measure each output-copy tolerance is checked on: per (sequence,
    head) (rel_err) for fp32 and bf16 checkpoints; for the E4M3 copy, whose 3
    mantissa bits alone can cost a single output vector more than the
    tolerance, the step's whole output (rel_err_step)."""
    return rel_err_step(y, ref) if copy_dtype == rs.RS_E4M3 else rel_err(y, ref)


def torch_dtype(code):
    return {rs.RS_F32: torch.float32, rs.RS_BF16: torch.bfloat16}[code]


# ------------------------------------------------------------------ Mamba-2

class Mamba2Case:
    """A Mamba-2 workload: params, an input stream, and oracle bookkeeping for a
    set of sampled (sequence, head) pairs (all pairs when `pairs` is None)."""

    def __init__(self, B, H, P, N, G, in_dtype, seed, device, pairs=None, gen_device=None):
        self.B, self.H, self.P, self.N, self.G = B, H, P, N, G
        self.device = torch.device(device)
        gdev = torch.device(gen_device or "cpu")
        self.A, self.D, dtb = gen.mamba2_params(H, seed + PARAM_SEED_OFFSET, gdev)
        self.stream = gen.Mamba2Stream(B, H, P, N, G, torch_dtype(in_dtype), dtb,
                                       seed + STREAM_SEED_OFFSET, gdev)
        self.pairs = [(b, h) for b in range(B) for h in range(H)] if pairs is None else list(pairs)
        self.pb = np.array([p[0] for p in self.pairs])
        self.ph = np.array([p[1] for p in self.pairs])
        self.pg = self.ph // (H // G)
        self.hstate = np.zeros((len(self.pairs), P, N))

    def draw(self, T):
        s = self.stream.next(T)
        return {k: v.to(self.device) for k, v in s.items()}

    def pair_inputs(self, s):
        """Oracle view of step dict s: per pair arrays [n, T, ...] in float64."""
        x = f64(s["x"])[:, self.pb, self.ph, :].transpose(1, 0, 2)
        dt = f64(s["dt"])[:, self.pb, self.ph].T
        Bm = f64(s["B"])[:, self.pb, self.pg, :].transpose(1, 0, 2)
        C = f64(s["C"])[:, self.pb, self.pg, :].transpose(1, 0, 2)
        return x, dt, Bm, C

    def oracle_run(self, s, advance=True, h=None):
        """Eager fp64 outputs [T, n, P] for the pairs; advances the oracle state."""
        x, dt, Bm, C = self.pair_inputs(s)
        A = f64(self.A)[self.ph]
        D = f64(self.D)[self.ph]
        h0 = (self.hstate if h is None else h).copy()
        y, h1 = oracle.mamba2_eager_batch(A, D, x, dt, Bm, C, h=h0)
        if advance and h is None:
            self.hstate = h1
        return y.transpose(1, 0, 2), h1

    def gpu_pairs(self, y):
        """y [..., B, H, R] tensor -> [..., n, R] numpy (sampled pairs)."""
        return f64(y)[..., self.pb, self.ph, :]


# ---------------------------------------------------------------------- GDN

class GdnCase:
    def __init__(self, B, H, dk, dv, in_dtype, seed, device, pairs=None, gen_device=None,
                 scale=1.0):
        self.B, self.H, self.dk, self.dv = B, H, dk, dv
        self.scale = scale
        self.device = torch.device(device)
        gdev = torch.device(gen_device or "cpu")
        A_log, dtb = gen.gdn_params(H, seed + PARAM_SEED_OFFSET, gdev)
        self.stream = gen.GdnStream(B, H, dk, dv, torch_dtype(in_dtype), A_log, dtb,
                                    seed + STREAM_SEED_OFFSET, gdev)
        self.pairs = [(b, h) for b in range(B) for h in range(H)] if pairs is None else list(pairs)
        self.pb = np.array([p[0] for p in self.pairs])
        self.ph = np.array([p[1] for p in self.pairs])
        self.hstate = np.zeros((len(self.pairs), dv, dk))

    def draw(self, T):
        s = self.stream.next(T)
        return {k: v.to(self.device) for k, v in s.items()}

    def pair_inputs(self, s):
        q = f64(s["q"])[:, self.pb, self.ph, :].transpose(1, 0, 2)
        k = f64(s["k"])[:, self.pb, self.ph, :].transpose(1, 0, 2)
        v = f64(s["v"])[:, self.pb, self.ph, :].transpose(1, 0, 2)
        a = f64(s["alpha"])[:, self.pb, self.ph].T
        b = f64(s["beta"])[:, self.pb, self.ph].T
        return q, k, v, a, b

    def oracle_run(self, s, advance=True, h=None):
        q, k, v, a, b = self.pair_inputs(s)
        h0 = (self.hstate if h is None else h).copy()
        o, h1 = oracle.gdn_eager_batch(q, k, v, a, b, S=h0, scale=self.scale)
        if advance and h is None:
            self.hstate = h1
        return o.transpose(1, 0, 2), h1

    def gpu_pairs(self, y):
        return f64(y)[..., self.pb, self.ph, :]


# ----------------------------------------------- quantised checkpoints ----

def dequantised(S, copy_dtype):
    """What a kernel reading the low-precision copy of fp32 master S sees, in
    fp64: bf16 RNE, or E4M3 codes x the per-tile scale (absmax / 448)."""
    S32 = np.asarray(S, np.float64).astype(np.float32)
    if copy_dtype == rs.RS_BF16:
        return oracle.bf16_decode(oracle.bf16_rne(S32)).astype(np.float64)
    if copy_dtype == rs.RS_E4M3:
        out = np.empty(S32.shape, np.float64)
        for i in range(S32.shape[0]):
            codes, scale = oracle.e4m3_quantize_tile(S32[i])
            out[i] = oracle.e4m3_decode(codes).astype(np.float64) * np.float64(np.float32(scale))
        return out
    return S32.astype(np.float64)


class QuantCheckpoint:
    """Oracle bookkeeping of the method's checkpoint for a low-precision arm.

    Outputs are replayed from the dequantised copy of the checkpoint plus the
    inputs buffered since it ("ReplaySSM: Cache SSM Inputs, Not State",
    Abstract: outputs come from the checkpoint and the cached inputs).  A
    commit of the dual-precision arm folds the buffer into the fp64 checkpoint;
    the shared arm has no master, so its commit folds the buffer into the
    dequantised copy, which is then quantised again."""

    def __init__(self, case, copy_dtype, shared):
        self.case, self.copy_dtype, self.shared = case, copy_dtype, shared
        self.ckpt = case.hstate.copy()
        self.buf = []

    def _cat(self):
        return {k: torch.cat([d[k] for d in self.buf], 0) for k in self.buf[0]}

    def step(self, s):
        """Appends step s; returns its expected outputs [T_s, n, R]."""
        self.buf.append(s)
        T = next(iter(s.values())).shape[0]
        y, _ = self.case.oracle_run(self._cat(), h=dequantised(self.ckpt, self.copy_dtype))
        return y[-T:]

    def commit(self):
        start = dequantised(self.ckpt, self.copy_dtype) if self.shared else self.ckpt
        _, self.ckpt = self.case.oracle_run(self._cat(), h=start)
        self.buf = []


# -------------------------------------------------------------- checks ----

def check_copy_is_quantised_master(sess):
    """No drift: the output copy is exactly the quantisation of the fp32 master
    (bf16 RNE, or E4M3 with scale = absmax / 448 per tile)."""
    cfg = sess.cfg
    master = sess.master().detach().cpu().numpy().astype(np.float32)
    if cfg.copy_dtype == rs.RS_BF16:
        got = sess.copy().detach().cpu().view(torch.int16).numpy().view(np.uint16)
        exp = oracle.bf16_rne(master)
        assert np.array_equal(got, exp), f"{np.sum(got != exp)} bf16 codes differ"
    elif cfg.copy_dtype == rs.RS_E4M3:
        codes = sess.copy().detach().cpu().numpy()
        scales = sess.scale().detach().cpu().numpy()
        B, H = master.shape[:2]
        for b in range(B):
            for h in range(H):
                c_exp, s_exp = oracle.e4m3_quantize_tile(master[b, h])
                assert scales[b, h] == s_exp, (b, h, scales[b, h], s_exp)
                assert np.array_equal(codes[b, h], c_exp), (b, h)


def make_session(kind, B, H, R, CC, G=1, cap=16, npos_max=1, in_dtype=rs.RS_BF16,
                 copy_dtype=rs.RS_BF16, out_dtype=rs.RS_F32, shared_lowp=0, A=None, D=None,
                 gdn_scale=1.0, device="cuda"):
    cfg = rs.make_config(kind, B, H, R, CC, G, cap, npos_max, in_dtype, copy_dtype, out_dtype,
                         shared_lowp, gdn_scale)
    return rs.ReplaySSM(cfg, A=A, D=D, device=device)
