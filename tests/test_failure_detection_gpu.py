"""A wait that nothing ever satisfies gives up within its limit, is reported as FA_ERR_TIMEOUT
through the device status word, and leaves the context usable (no trap, no hang)."""
import time

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import exact_attention_158_b200 as fa
    assert fa.device_status() == 0
    t0 = time.perf_counter()
    assert fa.selftest_wait_timeout(50_000) == 5  # FA_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 30
    assert fa.device_status() == 0  # cleared by the read
    # the context still runs the real kernels correctly afterwards
    case = W.PrefillCase("after", 1, 2, 300, 64, True)
    q, k, v = W.make_prefill(case, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.device_status() == 0 and torch.isfinite(o).all()


def test_selftest_rejects_bad_limits():
    import exact_attention_158_b200 as fa
    lib = fa.load_library()
    lib.fa_selftest_wait_timeout.argtypes = [__import__("ctypes").c_uint, __import__("ctypes").c_void_p]
    assert lib.fa_selftest_wait_timeout(0, None) == 1
    assert lib.fa_selftest_wait_timeout(3_000_000, None) == 1
