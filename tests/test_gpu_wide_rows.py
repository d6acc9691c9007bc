"""Speculative verification at the widest and narrowest supported state rows:
256 columns (16 k-steps of the tensor-core contraction and of the GDN prep's
Gram products, three consumer teams) and 16 columns (a single k-step), for
both layer kinds, against the fp64 oracle as in the ring-width rounds."""
import pytest

import rs_decode_outputs_b200 as rs
from tests.harness import TOL_BF16
from tests.test_gpu_ring_widths import setup, verify_rounds

pytestmark = pytest.mark.gpu

SHAPES = [
    # kind, R, CC, G, cap, npos
    ("gdn", 32, 256, 1, 16, 5),
    ("gdn", 48, 16, 1, 8, 5),
    ("m2", 32, 256, 1, 8, 5),
    ("m2", 64, 16, 2, 16, 8),
]


@pytest.mark.parametrize("kind,R,CC,G,cap,npos", SHAPES,
                         ids=[f"{k}-R{r}-C{c}-cap{cp}-n{n}" for k, r, c, _, cp, n in SHAPES])
def test_verify_rounds_at_row_width_limits(cuda_device, kind, R, CC, G, cap, npos):
    case, sess = setup(kind, R, CC, G, cap, npos, cuda_device, seed=1100 + R + CC, scale=0.5)
    verify_rounds(case, sess, kind, cap, npos, R, cuda_device, TOL_BF16)
