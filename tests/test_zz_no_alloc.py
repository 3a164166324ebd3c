"""The backward entry point that allocates nothing (axis_attn_bwd_noalloc).

Some callers cannot allocate device memory at the point where they run the
backward (inside an allocator callback, with a memory pool reserved up front,
or on a path that must not block on the allocator) and have no workspace to
hand over.  For them the library keeps a fixed 32 MiB scratch array of its own.
This test calls that entry point through the C ABI three times in a row (a
larger problem, a smaller one, the larger one again) and checks each result
against the ordinary entry point (caller-provided workspace) with the parity
tolerance of the other GPU tests.  The later calls check that what an earlier
call left in the shared scratch does not leak into the next result.  It also checks the size limit.

Kept in its own file, named to be collected last.
"""
import ctypes
import math

import pytest
import torch

import causal_attention_fwd_b200 as aa
from causal_attention_fwd_b200.synthetic import make_inputs

pytestmark = pytest.mark.gpu

TOL_GRAD = 1e-2
LIMIT = 32 << 20


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_fwd_b200 import build

    build.build()


def _noalloc(q, k, v, o, lse, do, causal, sc, stream):
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = aa.axis_attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                  lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  B, Hq, Hkv, S, D, sc, int(causal), stream)
    assert rc == 0, aa.axis_attn_strerror(rc)
    return dq, dk, dv


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / b.norm())


def test_noalloc_matches_workspace_entry_point_in_a_row():
    dev = torch.device("cuda:0")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # the larger problem, a smaller one with other region boundaries, then the
    # larger one again: nothing the smaller call left in the shared scratch may
    # leak into the third result
    problems = [(2, 12, 4, 1024, 64, True, 31), (1, 4, 2, 777, 128, False, 32), (2, 12, 4, 1024, 64, True, 31)]
    first = None
    for n, (B, Hq, Hkv, S, D, causal, seed) in enumerate(problems):
        assert aa.axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D) <= LIMIT
        sc = 1.0 / math.sqrt(D)
        q, k, v, do = (t.to(dev) for t in make_inputs(B, Hq, Hkv, S, D, seed))
        o, lse = aa.attention_forward(q, k, v, causal=causal, scale=sc)
        ref = aa.attention_backward(q, k, v, o, lse, do, causal=causal, scale=sc)
        got = _noalloc(q, k, v, o, lse, do, causal, sc, stream)
        aa.check_status()
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            assert torch.isfinite(g.float()).all(), name
            assert _rel(g, r) <= TOL_GRAD, (name, _rel(g, r))
        # dK and dV take no cross-CTA additions: the same kernels give the same bits
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
        if n == 0:
            first = got
        elif n == 2:
            assert torch.equal(got[1], first[1]) and torch.equal(got[2], first[2])
            assert _rel(got[0], first[0]) <= TOL_GRAD


def test_noalloc_rejects_sizes_beyond_the_scratch():
    # B=4, Hq=32, S=2048, D=64 needs ~69 MB of scratch: refused before any launch
    assert aa.axis_attn_bwd_workspace_bytes(4, 32, 8, 2048, 64) > LIMIT
    A = 1 << 20
    rc = aa.axis_attn_bwd_noalloc(*([A] * 9), 4, 32, 8, 2048, 64, 0.125, 1, None)
    assert rc == 5  # AXIS_ATTN_ERR_WORKSPACE
