"""fa_bwd (tcgen05 backward kernel) against the fp64 oracle's backward, on the forward's own O and
LSE and a seeded dO."""
import pytest
import torch

import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 257, 1000])
def test_backward_ragged(N, causal, d):
    parity.run_backward(W.PrefillCase(f"bwd_N{N}", 1, 2, N, d, causal))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_multi_tile(causal):
    # 8 key blocks per head, each streaming up to 8 query blocks through the 2-stage rings
    parity.run_backward(W.PrefillCase("bwd_multi", 2, 3, 1024, 128, causal))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_persistent_odd_key_blocks(causal, d):
    # N = 300: three key blocks per head (the middle pair is a single sub-unit, the last block is
    # ragged); 160 heads make 320 pairs, so each of the persistent CTAs walks two or three pairs
    # and carries its barrier phases across sub-units of different lengths.  Heads spread over
    # the CTAs are checked in full.
    parity.run_backward(W.PrefillCase(f"bwd_pers_d{d}", 4, 40, 300, d, causal),
                        heads=[0, 1, 73, 148, 149, 159])


@pytest.mark.parametrize("causal", [False, True])
def test_backward_config_sampled_heads(causal):
    # the bench's training-shape configuration (B8 H16 N2048 d128), three heads checked in full
    parity.run_backward(W.PrefillCase("bwd_prefill", 8, 16, 2048, 128, causal), heads=[0, 77, 127])


@pytest.mark.parametrize("d", [64, 128])
def test_backward_bf16_grads(d):
    parity.run_backward(W.PrefillCase("bwd_bf16", 1, 2, 700, d, True), grad_dtype=torch.bfloat16)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 33, 129, 257, 1000])
def test_backward_ragged_bf16_grads(N, causal):
    # bf16 dK / dV, rows past N never written
    parity.run_backward(W.PrefillCase(f"bwd_bf16_N{N}", 1, 3, N, 128, causal),
                        grad_dtype=torch.bfloat16)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_peaked_rows_f32_o(d):
    # 1% of key rows x8: near one-hot probability rows.  There D = dO . O cancels against the
    # dominant dP, so O's own bf16 rounding would dominate dQ's error; the forward's fp32 O is used.
    parity.run_backward(W.PrefillCase("bwd_peaked", 1, 4, 1024, d, True, peaked=True),
                        o_dtype=torch.float32)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_f32_o(causal):
    parity.run_backward(W.PrefillCase("bwd_o32", 1, 2, 1000, 128, causal), o_dtype=torch.float32)


def test_backward_scale_override():
    parity.run_backward(W.PrefillCase("bwd_scale", 1, 2, 300, 128, False), scale=0.3)


def test_dk_dv_deterministic_dq_stable():
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("bwd_det", 2, 2, 777, 128, True)
    q, k, v = W.make_prefill(case, device="cuda")
    do = W.make_dout(case, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=True)
    a = fa.fa_bwd(q, k, v, o, do, lse, causal=True, grad_dtype=torch.float32)
    b = fa.fa_bwd(q, k, v, o, do, lse, causal=True, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dQ partials are added in whatever order the key blocks finish: equal up to fp32 reordering
    assert (a[0] - b[0]).abs().max().item() <= 1e-5 * a[0].abs().max().item()


def test_guard_bytes_untouched():
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("bwd_guard", 1, 2, 200, 64, False)
    q, k, v = W.make_prefill(case, device="cuda")
    do = W.make_dout(case, device="cuda")
    o, lse = fa.fa_fwd(q, k, v)
    lib = fa.load_library()
    n = q.numel()
    pad = 256
    bufs = [torch.full((n + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
            for _ in range(3)]
    ws = torch.empty(lib.fa_bwd_workspace_size(1, 2, 200, 64), dtype=torch.uint8, device="cuda")
    st = lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), 0, do.data_ptr(),
                    lse.data_ptr(), *(b[pad:].data_ptr() for b in bufs), 1, 1, 2, 200, 64, 0, 0.0,
                    ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and fa.device_status() == 0
    for b in bufs:
        assert torch.isnan(b[:pad]).all() and torch.isnan(b[pad + n:]).all()
        assert torch.isfinite(b[pad:pad + n]).all()


@pytest.mark.parametrize("d", [64, 128])
def test_guard_bytes_untouched_bf16_grads(d):
    # bf16 gradients written into the middle of NaN-filled buffers: nothing outside [B, H, N, d]
    # changes, also where a key block's last 32-row box reaches past N
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("bwd_guard_bf16", 1, 2, 200, d, False)
    q, k, v = W.make_prefill(case, device="cuda")
    do = W.make_dout(case, device="cuda")
    o, lse = fa.fa_fwd(q, k, v)
    n = q.numel()
    pad = 4096
    bufs = [torch.full((n + 2 * pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
            for _ in range(3)]
    views = [b[pad:pad + n].view(q.shape) for b in bufs]
    lib = fa.load_library()
    ws = torch.empty(lib.fa_bwd_workspace_size(1, 2, 200, d), dtype=torch.uint8, device="cuda")
    st = lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), 0, do.data_ptr(),
                    lse.data_ptr(), *(t.data_ptr() for t in views), 0, 1, 2, 200, d, 0, 0.0,
                    ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and fa.device_status() == 0
    for b in bufs:
        assert torch.isnan(b[:pad]).all() and torch.isnan(b[pad + n:]).all()
        assert torch.isfinite(b[pad:pad + n]).all()
