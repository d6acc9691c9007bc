"""Schedule models for ReplaySSM -- TEST INFRASTRUCTURE (see ``oracle/__init__``).

Two models, both written from the pages' description of the method:

``RingPointers``
    The integer bookkeeping of the input buffer: per sequence a head (the
    position the checkpoint stands at) and a tail (one past the newest buffered
    input), as monotonically increasing logical positions; ``len = tail - head``.
    "ReplaySSM for hybrid SSM-Transformer stacks", How ReplaySSM works:
    step 2 appends each new SSM input to the buffer; step 3 folds the buffer
    into the checkpoint and resets the buffer (here: head <- tail); step 4
    rejects the last k speculative tokens by moving the tail pointer back by k,
    leaving the checkpoint untouched.  Data-dependent misuse (overflowing the
    ring, rolling back more than is buffered, reading an empty buffer) leaves the
    pointers unchanged and sets a sticky per-sequence error bit.

``Mamba2Replay`` / ``GdnReplay``
    One (sequence, head) in fp64: a checkpoint plus the list of buffered
    inputs.  ``output()`` replays the buffer against the checkpoint without
    forming any state (Abstract: output computation separated from checkpoint
    updates); ``commit()`` applies the recurrence across the buffer and makes the
    result the new checkpoint (step 3); ``rollback(k)`` forgets the last k inputs
    (step 4).  Used to pin the invariants: replay equals eager, commit-then-
    continue equals never committing, rollback equals recomputing the truncated
    input.
"""
import numpy as np

from . import gdn_eager, gdn_replay, mamba2_eager, mamba2_replay

# Sticky per-sequence error bits (values are part of the library's C interface).
ERR_OVERFLOW = 1    # append would exceed the ring capacity
ERR_ROLLBACK = 2    # rollback count outside [0, len]
ERR_EMPTY = 4       # output requested with fewer buffered entries than positions


class RingPointers:
    def __init__(self, batch: int, cap: int):
        self.cap = int(cap)
        self.head = np.zeros(batch, dtype=np.int64)
        self.tail = np.zeros(batch, dtype=np.int64)
        self.err = np.zeros(batch, dtype=np.uint32)

    @property
    def length(self):
        return self.tail - self.head

    def append(self, T: int):
        ok = self.length + T <= self.cap
        self.tail = np.where(ok, self.tail + T, self.tail)
        self.err |= np.where(ok, 0, ERR_OVERFLOW).astype(np.uint32)

    def rollback(self, k):
        k = np.broadcast_to(np.asarray(k, dtype=np.int64), self.tail.shape)
        ok = (k >= 0) & (k <= self.length)
        self.tail = np.where(ok, self.tail - k, self.tail)
        self.err |= np.where(ok, 0, ERR_ROLLBACK).astype(np.uint32)

    def commit(self, min_len: int = 1, mask=None):
        sel = self.length >= max(int(min_len), 1)
        if mask is not None:
            sel &= np.asarray(mask).astype(bool)
        self.head = np.where(sel, self.tail, self.head)
        return sel

    def check_outputs(self, npos: int):
        """Outputs at the newest ``npos`` positions need len >= npos."""
        bad = self.length < npos
        self.err |= np.where(bad, ERR_EMPTY, 0).astype(np.uint32)
        return ~bad

    def slots(self, b: int):
        """Ring slots of sequence b's buffered entries, oldest first."""
        return [int(p) % self.cap for p in range(int(self.head[b]), int(self.tail[b]))]


class Mamba2Replay:
    def __init__(self, A, D, S0):
        self.A, self.D = float(A), float(D)
        self.S0 = np.array(S0, dtype=np.float64)
        self.x, self.dt, self.B, self.C = [], [], [], []

    def append(self, x, dt, B, C):
        self.x.append(np.asarray(x, np.float64))
        self.dt.append(float(dt))
        self.B.append(np.asarray(B, np.float64))
        self.C.append(np.asarray(C, np.float64))

    def __len__(self):
        return len(self.x)

    def output(self, upto=None):
        """Output at buffered position ``upto`` (default: the newest)."""
        n = len(self.x) if upto is None else upto + 1
        return mamba2_replay(self.A, self.D, self.S0, np.stack(self.x[:n]),
                             np.array(self.dt[:n]), np.stack(self.B[:n]), np.stack(self.C[:n]))

    def commit(self):
        if self.x:
            _, self.S0 = mamba2_eager(self.A, self.D, np.stack(self.x), np.array(self.dt),
                                      np.stack(self.B), np.stack(self.C), h0=self.S0)
        self.x, self.dt, self.B, self.C = [], [], [], []

    def rollback(self, k: int):
        if not 0 <= k <= len(self.x):
            raise ValueError("rollback beyond the buffer")
        n = len(self.x) - k
        self.x, self.dt, self.B, self.C = self.x[:n], self.dt[:n], self.B[:n], self.C[:n]


class GdnReplay:
    def __init__(self, S0, scale=1.0):
        self.scale = float(scale)
        self.S0 = np.array(S0, dtype=np.float64)
        self.q, self.k, self.v, self.alpha, self.beta = [], [], [], [], []

    def append(self, q, k, v, alpha, beta):
        self.q.append(np.asarray(q, np.float64))
        self.k.append(np.asarray(k, np.float64))
        self.v.append(np.asarray(v, np.float64))
        self.alpha.append(float(alpha))
        self.beta.append(float(beta))

    def __len__(self):
        return len(self.k)

    def output(self, upto=None):
        n = len(self.k) if upto is None else upto + 1
        return gdn_replay(self.S0, np.stack(self.k[:n]), np.stack(self.v[:n]),
                          np.array(self.alpha[:n]), np.array(self.beta[:n]), self.q[n - 1],
                          scale=self.scale)

    def commit(self):
        if self.k:
            _, self.S0 = gdn_eager(np.stack(self.q), np.stack(self.k), np.stack(self.v),
                                   np.array(self.alpha), np.array(self.beta), S0=self.S0,
                                   scale=self.scale)
        self.q, self.k, self.v, self.alpha, self.beta = [], [], [], [], []

    def rollback(self, k: int):
        if not 0 <= k <= len(self.k):
            raise ValueError("rollback beyond the buffer")
        n = len(self.k) - k
        self.q, self.k, self.v = self.q[:n], self.k[:n], self.v[:n]
        self.alpha, self.beta = self.alpha[:n], self.beta[:n]
