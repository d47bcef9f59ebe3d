"""fa_fwd (tcgen05 prefill kernel) against the fp64 oracle on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_tiny(causal, out_dtype):
    parity.run_prefill(W.PrefillCase("tiny", 1, 1, 256, 64, causal), out_dtype, full=True)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 256, 257, 383, 1000])
def test_ragged_lengths(N, causal, d):
    parity.run_prefill(W.PrefillCase(f"ragged_N{N}", 2, 2, N, d, causal), torch.float32, full=True)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 31, 32, 33, 129, 255, 1000])
def test_ragged_lengths_bf16_out(N, causal, d):
    # bf16 O: at d = 128 it leaves through tensor stores of 32-row boxes, clipped at row N
    parity.run_prefill(W.PrefillCase(f"ragged_bf16_N{N}", 2, 3, N, d, causal), torch.bfloat16,
                       full=True)


@pytest.mark.parametrize("causal", [False, True])
def test_multi_tile_full(causal):
    # several heads, 8 query pairs, 16 key blocks: exercises the ring, the persistent loop and
    # the causal pairing of work units, every row checked
    parity.run_prefill(W.PrefillCase("multi", 2, 3, 2048, 128, causal), torch.float32, full=True)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_prefill_config(causal, out_dtype):
    # B=8, H=16, N=2048, d=128: the launch configuration the bench times; sampled rows
    parity.run_prefill(W.PrefillCase("prefill", 8, 16, 2048, 128, causal), out_dtype)


@pytest.mark.parametrize("shape", [(8, 16, 2048, 128), (32, 16, 512, 128), (4, 16, 4096, 128)],
                         ids=lambda s: "B{}H{}N{}d{}".format(*s))
def test_scheduled_causal_writes_every_row(shape):
    # causal launches of these shapes run their units from a host-built table (fa_fwd_schedule):
    # every row must be written (the outputs start as NaN), and row 0 of each head, which sees key
    # 0 alone, is V's row 0 with LSE = scale * q_0 . k_0
    import math
    import exact_attention_158_b200 as fa
    B, H, N, d = shape
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert fa.fwd_schedule(B, H, N, d, sms) is not None
    q, k, v = W.make_prefill(W.PrefillCase("sched", B, H, N, d, True), device="cuda")
    o = torch.full((B, H, N, d), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    fa.fa_fwd(q, k, v, causal=True, out_dtype=torch.float32, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all(), "a unit was never run"
    torch.testing.assert_close(o[:, :, 0, :], v[:, :, 0, :].float(), rtol=1e-6, atol=1e-6)
    s00 = (q[:, :, 0, :].double() * k[:, :, 0, :].double()).sum(-1) / math.sqrt(d)
    torch.testing.assert_close(lse[:, :, 0].double(), s00, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("case", W.sweep_cases(128) + W.sweep_cases(64),
                         ids=lambda c: f"{c.name}_N{c.N}_{'causal' if c.causal else 'full'}")
def test_sweep(case):
    parity.run_prefill(case, torch.float32)


@pytest.mark.parametrize("case", [c for c in W.sweep_cases(64) if c.N in (512, 4096)],
                         ids=lambda c: f"{c.name}_N{c.N}_{'causal' if c.causal else 'full'}")
def test_sweep_bf16_out(case):
    parity.run_prefill(case, torch.bfloat16)


def test_peaked_rows_full_small():
    # 1% of key rows scaled x8 gives peaked softmax rows: full check on a small shape
    parity.run_prefill(W.PrefillCase("peaked", 2, 4, 1024, 64, True, peaked=True), torch.float32,
                       full=True)


def test_scale_override_and_aliasing():
    import exact_attention_158_b200 as fa
    from oracle import oracle as orc
    case = W.PrefillCase("alias", 1, 2, 300, 128, False)
    q, _, _ = W.make_prefill(case, device="cuda")
    o, lse = fa.fa_fwd(q, q, q, causal=False, scale=0.05, out_dtype=torch.float32)
    qb = W.bf16_bits(q).reshape(2, 300, 128)
    o_ref, lse_ref = orc.attention(qb, qb, qb, False, 0.05)
    parity.assert_close(o.cpu().numpy().reshape(2, 300, 128), lse.cpu().numpy().reshape(2, 300),
                        o_ref, lse_ref, "q=k=v, scale 0.05")


def test_guard_bytes_untouched():
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("guard", 1, 3, 200, 64, True)
    q, k, v = W.make_prefill(case, device="cuda")
    n = 3 * 200 * 64
    pad = 4096
    buf = torch.full((n + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
    lbuf = torch.full((3 * 200 + 2 * pad,), float("nan"), dtype=torch.float32, device="cuda")
    o = buf[pad:pad + n].view(1, 3, 200, 64)
    lse = lbuf[pad:pad + 600].view(1, 3, 200)
    fa.fa_fwd(q, k, v, causal=True, out_dtype=torch.float32, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[pad + n:]).all()
    assert torch.isnan(lbuf[:pad]).all() and torch.isnan(lbuf[pad + 600:]).all()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("d", [64, 128])
def test_guard_bytes_untouched_bf16_out(d):
    # bf16 O written into the middle of a NaN-filled buffer: nothing outside [B, H, N, d] changes,
    # also where the last 32-row box of a head reaches past N
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("guard_bf16", 1, 3, 200, d, False)
    q, k, v = W.make_prefill(case, device="cuda")
    n = 3 * 200 * d
    pad = 4096
    buf = torch.full((n + 2 * pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    o = buf[pad:pad + n].view(1, 3, 200, d)
    fa.fa_fwd(q, k, v, causal=False, out_dtype=torch.bfloat16, out=o)
    torch.cuda.synchronize()
    assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[pad + n:]).all()
    assert torch.isfinite(o).all()


def test_repeatable_bitwise():
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("rep", 2, 4, 1024, 128, True)
    q, k, v = W.make_prefill(case, device="cuda")
    o1, l1 = fa.fa_fwd(q, k, v, causal=True)
    o2, l2 = fa.fa_fwd(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_long_sequence_128k(causal):
    # one head pair over N = 131072 (1024 key blocks per row tile, 256 query-tile pairs per head):
    # sampled rows, including the last ones, against the oracle
    parity.run_prefill(W.PrefillCase("long_128k", 1, 2, 131072, 128, causal), torch.float32)


def test_many_heads_short_rows():
    # B*H = 4096 (b, h) slices of N = 129: many units, each a full tile plus a one-row tile
    parity.run_prefill(W.PrefillCase("many_heads", 64, 64, 129, 64, True), torch.float32)
