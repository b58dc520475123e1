"""The device-side timeout path, exercised without faulting or hanging the GPU.

lh_selftest_wait_timeout launches the attention forward kernel with its TMA
producer told to load nothing and a short bound on every barrier wait: the
MMA and softmax warps wait on barriers that never complete, the first wait to
run out stops every role, and the kernel returns with the timeout bit set in
the error word.  No copy or MMA was issued, so nothing is in flight when the
waits give up.  The test checks the status, that the kernel returned well
within its bound, and that the context still runs a normal call correctly."""

import ctypes
import time

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_pyramid_b200 as lh
from hierarchical_sparse_attention_pyramid_b200 import _lib
from oracle import lighthouse_oracle as lo
from tests import parity_util as pu

LH_ERR_TIMEOUT = 5


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_bounded_wait_runs_out_and_reports_timeout():
    lib = _lib.load()
    ws = torch.zeros(_lib.SELFTEST_WS_BYTES, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    for cycles in (2_000_000, 20_000_000):  # about 1 ms and 10 ms at the boost clock
        t0 = time.perf_counter()
        _lib.call("lh_selftest_wait_timeout", ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(ws.numel()),
                  ctypes.c_int64(cycles), _stream())
        status = lib.lh_check_error(ctypes.c_void_p(ws.data_ptr()), _stream())  # synchronises the stream
        elapsed = time.perf_counter() - t0
        assert status == LH_ERR_TIMEOUT, _lib.STATUS_NAMES.get(status, status)
        assert elapsed < 2.0, elapsed
        # lh_check_error cleared the word
        assert lib.lh_check_error(ctypes.c_void_p(ws.data_ptr()), _stream()) == 0


@pytest.mark.gpu
def test_context_usable_after_timeout():
    lib = _lib.load()
    ws = torch.zeros(_lib.SELFTEST_WS_BYTES, dtype=torch.uint8, device="cuda")
    _lib.call("lh_selftest_wait_timeout", ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(ws.numel()),
              ctypes.c_int64(2_000_000), _stream())
    assert lib.lh_check_error(ctypes.c_void_p(ws.data_ptr()), _stream()) == LH_ERR_TIMEOUT
    g = torch.Generator().manual_seed(77)
    q, k, v = (torch.randn(1, 300, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    L = lh.Layer(1, 1, 4096, 64, 3, 2, 8)
    os_, lse = lh.attn_fwd(L, q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    O, ls = lo.causal_attention(pu.to_np(q[0]), pu.to_np(k[0]), pu.to_np(v[0]))
    pu.assert_close(os_[0], O, "O after a timed-out launch")
    np.testing.assert_allclose(pu.to_np(lse[0]), ls, rtol=1e-4, atol=1e-4)
