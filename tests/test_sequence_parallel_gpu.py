"""Key-range partials (fa_fwd_keyrange) and their merge (fa_merge_partials) against the fp64
oracle; the sequence-sharded forward emulated on one GPU as one launch per key range."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def bits(t):
    return W.bf16_bits(t)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("q_row0,k_lo,k_hi", [(0, 0, 300), (0, 300, 301), (0, 301, 1000),
                                              (200, 129, 700), (999, 0, 1000)])
def test_keyrange_partial(d, causal, q_row0, k_lo, k_hi):
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("kr", 1, 2, 1000, d, causal)
    q, k, v = W.make_prefill(case, device="cuda")
    kr, vr = k[:, :, k_lo:k_hi].contiguous(), v[:, :, k_lo:k_hi].contiguous()
    o = torch.full(q.shape, 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full(q.shape[:3], 7.0, dtype=torch.float32, device="cuda")
    fa.fa_fwd_keyrange(q, kr, vr, q_row0=q_row0, k_pos0=k_lo, causal=causal, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    ro, rl = orc.attention_keyrange(bits(q)[:, :, q_row0:].copy(), bits(kr), bits(vr), q_row0, k_lo,
                                    causal, case.scale)
    og, lg = o[:, :, q_row0:].cpu().numpy(), lse[:, :, q_row0:].cpu().numpy()
    empty = np.isneginf(rl)
    assert np.array_equal(np.isneginf(lg), empty), "rows without visible keys must get LSE = -inf"
    assert np.all(og[empty] == 0.0)
    if (~empty).any():
        parity.assert_close(og[~empty], lg[~empty], ro[~empty], rl[~empty],
                            f"keyrange rows>={q_row0} keys[{k_lo},{k_hi})")
    # rows before q_row0 are untouched
    assert torch.all(o[:, :, :q_row0] == 7.0) and torch.all(lse[:, :, :q_row0] == 7.0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cuts", [[1000], [513, 1000], [1, 128, 700, 1000]])
def test_sharded_forward_emulated(d, causal, cuts):
    # one fa_fwd_keyrange launch per key range (the ranks of the sharded forward), then the merge
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("sp", 2, 2, 1000, d, causal)
    q, k, v = W.make_prefill(case, device="cuda")
    bounds = [0] + cuts
    parts_o, parts_l = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        po, pl = fa.fa_fwd_keyrange(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(),
                                    k_pos0=a, causal=causal)
        parts_o.append(po)
        parts_l.append(pl)
    o, lse = fa.fa_merge_partials(torch.stack(parts_o), torch.stack(parts_l),
                                  out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    ro, rl = orc.attention(bits(q), bits(k), bits(v), causal, case.scale)
    parity.assert_close(o.cpu().numpy(), lse.cpu().numpy(), ro, rl, f"sharded {cuts}")


def test_sharded_long_sequence_sampled():
    # B1 H16 N8192 d128 causal over four key ranges; sampled rows against the oracle
    import exact_attention_158_b200 as fa
    case = W.PrefillCase("sp_long", 1, 16, 8192, 128, True)
    q, k, v = W.make_prefill(case, device="cuda")
    parts = [fa.fa_fwd_keyrange(q, k[:, :, a:a + 2048].contiguous(), v[:, :, a:a + 2048].contiguous(),
                                k_pos0=a, causal=True) for a in range(0, 8192, 2048)]
    o, lse = fa.fa_merge_partials(torch.stack([p[0] for p in parts]),
                                  torch.stack([p[1] for p in parts]), out_dtype=torch.float32)
    torch.cuda.synchronize()
    pairs = parity.sample_rows(case)
    BH, N, d = 16, 8192, 128
    ro, rl = orc.attention_rows(bits(q).reshape(BH, N, d), bits(k).reshape(BH, N, d),
                                bits(v).reshape(BH, N, d), True, case.scale, pairs)
    og = o.reshape(BH, N, d)[pairs[:, 0], pairs[:, 1]].cpu().numpy()
    lg = lse.reshape(BH, N)[pairs[:, 0], pairs[:, 1]].cpu().numpy()
    parity.assert_close(og, lg, ro, rl, "sharded long sequence (sampled rows)")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_merge_kernel(d, out_dtype):
    import exact_attention_158_b200 as fa
    g = torch.Generator().manual_seed(11)
    G, rows = 5, 777
    op = torch.randn(G, rows, d, generator=g, dtype=torch.float64)
    lp = 30.0 * torch.randn(G, rows, generator=g, dtype=torch.float64)
    lp[1, ::3] = -float("inf")       # ranges without visible keys
    lp[:, 5] = -float("inf")         # a row that sees nothing anywhere
    op[1, ::3] = 0.0
    op[:, 5] = 0.0
    o, lse = fa.fa_merge_partials(op.float().cuda(), lp.float().cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    ro, rl = orc.merge_partials(op.float().double().numpy(), lp.float().double().numpy())
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    tol = 2.0 ** -8 if out_dtype == torch.bfloat16 else 1e-5
    assert np.all(og[5] == 0.0) and np.isneginf(lg[5])
    assert np.abs(og - ro).max() <= tol * max(1.0, np.abs(ro).max())
    fin = np.isfinite(rl)
    assert np.abs(lg[fin] - rl[fin]).max() <= 1e-4 * max(1.0, np.abs(rl[fin]).max())
