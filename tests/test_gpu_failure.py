"""The failure path of the kernels' bounded waits, exercised without a fault.

A test-only build of the library drops one phase of mbarrier arrives
(AXIS_ATTN_TEST_DROP_ARRIVE): in the forward, the softmax warps of the first
query tile never report their first P tile, so the P V issuer's wait cannot
complete; in the backward, the compute warps never report their first P^T /
dS^T tile, so the gradient-MMA issuer's wait cannot complete.  That one wait
site gets a short limit (2^22 SM clocks, about 2 ms; AXIS_ATTN_TEST_SHORT_SITE),
every other wait keeps the normal one.  Nothing faults and nothing spins
without bound: the waiting thread gives up at the limit, records the timeout
and its site, the other roles stop on the abort flag (other CTAs on the changed
timeout count), copies and MMAs in flight drain, TMEM is freed and the kernel
returns.  The test checks
that axis_attn_get_status() reports AXIS_ATTN_ERR_TIMEOUT with the expected
site, that a second launch of the same build reports its own timeout, and that
the ordinary library afterwards still gives oracle-exact results on the same
device (the CUDA context stayed usable).
"""
import ctypes
import math

import pytest
import torch

from causal_attention_fwd_b200.synthetic import make_inputs

from gpu_util import assert_close, run_gpu

pytestmark = pytest.mark.gpu

ERR_TIMEOUT = 7
SITE_FWD_PFULL = 5    # F_PFULL in attn_fwd.cuh
SITE_BWD_PDSFULL = 25  # B_PDSFULL in attn_bwd.cuh


@pytest.fixture(scope="module")
def fail_libs(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_fwd_b200 import build

    build.build()
    d = tmp_path_factory.mktemp("failbuild")
    libs = {}
    for mode in (1, 2):
        path = str(d / f"libaxis_attn_drop{mode}.so")
        site = SITE_FWD_PFULL if mode == 1 else SITE_BWD_PDSFULL
        build.build(force=True, out=path,
                    extra=[f"-DAXIS_ATTN_TEST_DROP_ARRIVE={mode}", f"-DAXIS_ATTN_TEST_SHORT_SITE={site}"])
        lib = ctypes.CDLL(path)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.axis_attn_fwd.argtypes = [vp] * 5 + [i] * 5 + [f, i, vp]
        lib.axis_attn_bwd.argtypes = [vp] * 9 + [i] * 5 + [f, i, vp, sz, vp]
        lib.axis_attn_bwd_workspace_bytes.argtypes = [i] * 5
        lib.axis_attn_bwd_workspace_bytes.restype = sz
        lib.axis_attn_get_status.argtypes = [vp]
        lib.axis_attn_last_status_word.restype = ctypes.c_uint
        libs[mode] = lib
    return libs


SHAPE = (1, 4, 2, 384, 64)  # B, Hq, Hkv, S, D: several tiles, several CTAs


def _tensors():
    B, Hq, Hkv, S, D = SHAPE
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in make_inputs(B, Hq, Hkv, S, D, seed=77))
    return q, k, v, do


def _expect_timeout(lib, site, stream):
    rc = lib.axis_attn_get_status(stream)
    word = lib.axis_attn_last_status_word()
    assert rc == ERR_TIMEOUT, rc
    assert word & 1 and (word >> 8) & 0xFF == site, hex(word)


def test_forward_wait_times_out_and_reports(fail_libs):
    lib = fail_libs[1]
    B, Hq, Hkv, S, D = SHAPE
    q, k, v, _ = _tensors()
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), device=q.device, dtype=torch.float32)
    sp = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):  # the second launch times out on its own, not on a stale report
        rc = lib.axis_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               B, Hq, Hkv, S, D, 1.0 / math.sqrt(D), 1, sp)
        assert rc == 0
        _expect_timeout(lib, SITE_FWD_PFULL, sp)
    assert lib.axis_attn_get_status(sp) == 0  # the report was cleared


def test_backward_wait_times_out_and_reports(fail_libs):
    import causal_attention_fwd_b200 as aa

    lib = fail_libs[2]
    B, Hq, Hkv, S, D = SHAPE
    sc = 1.0 / math.sqrt(D)
    q, k, v, do = _tensors()
    o, lse = aa.attention_forward(q, k, v, causal=True, scale=sc)  # ordinary library
    aa.check_status()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = lib.axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D)
    ws = torch.empty(wsb, device=q.device, dtype=torch.uint8)
    sp = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.axis_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                           lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, S, D,
                           sc, 1, ws.data_ptr(), wsb, sp)
    assert rc == 0
    _expect_timeout(lib, SITE_BWD_PDSFULL, sp)


def test_ordinary_library_still_exact_after_timeouts(fail_libs, oracle_mod):
    B, Hq, Hkv, S, D = SHAPE
    sc = 1.0 / math.sqrt(D)
    q, k, v, do = make_inputs(B, Hq, Hkv, S, D, seed=78)
    got = run_gpu(q, k, v, do, True, sc)
    ro, rl = oracle_mod.attn_fwd(q, k, v, sc, True)
    rdq, rdk, rdv, _ = oracle_mod.attn_bwd(q, k, v, do, sc, True)
    print(assert_close(*got, ro, rl, rdq, rdk, rdv, tag="after timeouts"))
