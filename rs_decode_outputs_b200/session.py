"""A handle plus the workspace it lives in, with torch views of its regions.

Thin convenience over the C interface: it allocates the workspace with torch
(the library itself never allocates device memory), keeps A / D alive for the
handle's lifetime, and exposes the checkpoint copies and pointers as tensor
views for inspection.  Every compute step is a call into the CUDA library.
"""
import torch

from . import _lib as L


class ReplaySSM:
    def __init__(self, cfg: L.RsConfig, A=None, D=None, device="cuda", stream=None):
        self.cfg = cfg
        self.layout = L.rs_workspace_layout(cfg)
        self.device = torch.device(device)
        self.workspace = torch.empty(self.layout.total, dtype=torch.uint8, device=self.device)
        self.A = None if A is None else A.to(self.device, torch.float32).contiguous()
        self.D = None if D is None else D.to(self.device, torch.float32).contiguous()
        self.handle = L.rs_create(cfg, self.workspace, self.A, self.D, stream)

    # ---------------------------------------------------------------- views
    def _view(self, off, nbytes, dtype, shape):
        if nbytes == 0:
            return None
        return self.workspace[off:off + nbytes].view(dtype).view(*shape)

    @property
    def tile_shape(self):
        c = self.cfg
        return (c.batch, c.nheads, c.headdim, c.dstate)

    def master(self):
        return self._view(self.layout.master, self.layout.master_bytes, torch.float32,
                          self.tile_shape)

    def copy(self):
        c = self.cfg
        if c.copy_dtype == L.RS_NONE:
            return None
        return self._view(self.layout.copy, self.layout.copy_bytes, L.TORCH_DTYPE[c.copy_dtype],
                          self.tile_shape)

    def scale(self):
        return self._view(self.layout.scale, self.layout.scale_bytes, torch.float32,
                          (self.cfg.batch, self.cfg.nheads))

    def head(self):
        return self._view(self.layout.head, 4 * self.cfg.batch, torch.int32, (self.cfg.batch,))

    def tail(self):
        return self._view(self.layout.tail, 4 * self.cfg.batch, torch.int32, (self.cfg.batch,))

    def err(self):
        return self._view(self.layout.err, 4 * self.cfg.batch, torch.int32, (self.cfg.batch,))

    # ---------------------------------------------------------------- calls
    def out_shape(self, npos=None):
        c = self.cfg
        base = (c.batch, c.nheads, c.headdim)
        return base if npos is None else (npos,) + base

    def new_out(self, npos=None):
        return torch.empty(self.out_shape(npos), dtype=L.TORCH_DTYPE[self.cfg.out_dtype],
                           device=self.device)

    def load_checkpoint(self, state, stream=None):
        L.rs_load_checkpoint(self.handle, state, stream)

    def append(self, inputs, T, stream=None):
        L.rs_append(self.handle, inputs, T, stream)

    def decode(self, y=None, stream=None):
        y = self.new_out() if y is None else y
        L.rs_decode_outputs(self.handle, y, stream)
        return y

    def decode_step(self, inputs, T=1, y=None, stream=None):
        """Append T inputs and return the outputs at those T positions."""
        y = self.new_out(None if T == 1 else T) if y is None else y
        L.rs_decode_step(self.handle, inputs, T, y, stream)
        return y

    def commit(self, min_len=1, mask=None, stream=None):
        L.rs_commit(self.handle, min_len, mask, stream)

    def verify(self, npos, y=None, stream=None):
        y = self.new_out(npos) if y is None else y
        L.rs_verify_outputs(self.handle, npos, y, stream)
        return y

    def rollback(self, k, stream=None):
        L.rs_rollback(self.handle, k, stream)

    def eager_step(self, state, state_dtype, inputs, T, y=None, stream=None):
        y = self.new_out(T) if y is None else y
        L.rs_eager_step(self.handle, state, state_dtype, inputs, T, y, stream)
        return y

    def eager_verify(self, slots, state_dtype, cur, inputs, npos, y=None, stream=None):
        y = self.new_out(npos) if y is None else y
        L.rs_eager_verify(self.handle, slots, state_dtype, cur, inputs, npos, y, stream)
        return y

    def eager_accept(self, cur, keep, stream=None):
        L.rs_eager_accept(self.handle, cur, keep, stream)

    def get_error(self, stream=None):
        return L.rs_get_error(self.handle, self.cfg.batch, stream)

    def clear_error(self, stream=None):
        L.rs_clear_error(self.handle, stream)

    def read_ptrs(self, stream=None):
        return L.rs_read_ptrs(self.handle, self.cfg.batch, stream)

    def close(self):
        if getattr(self, "handle", None) is not None:
            L.rs_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
