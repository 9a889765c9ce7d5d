"""Failure detection on the GPU without faulting it: a pipeline wait whose barrier
phase never completes ends, after its time limit, with SSTA_ERR_DEVICE_TIMEOUT in the
status word and an exited kernel; the context stays usable afterwards."""
import ctypes
import time

import pytest
import torch

import block_sparse_video_ssta_b200 as S
import ssta_inputs as si
from ssta_parity import full_check

pytestmark = pytest.mark.gpu

_f = S.lib.ssta_selftest_bounded_wait
_f.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
_f.restype = ctypes.c_int


def _run(timeout_us, complete):
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc = _f(timeout_us, complete, ctypes.c_void_p(ws.data_ptr()), 256,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, S.ssta_status_string(rc)
    code = S.ssta_read_device_status(ws)
    return code, time.perf_counter() - t0


def test_wait_that_never_completes_times_out(cuda_ok):
    code, secs = _run(20000, 0)                 # 20 ms limit
    assert code == 6 and S.ssta_status_string(code) == "SSTA_ERR_DEVICE_TIMEOUT"
    assert 0.015 <= secs < 2.0


def test_wait_that_completes_reports_nothing(cuda_ok):
    code, secs = _run(20000, 1)
    assert code == 0 and secs < 2.0


def test_context_usable_after_timeout(cuda_ok):
    assert _run(5000, 0)[0] == 6
    w = si.with_overrides(si.get_workload("small_bf16"), H=2, T=8, Y=16, X=16)
    st = full_check(w, seed=1)
    assert st["rows_mask_mismatch"] == 0
