"""fa_decode_paged (split-KV paged decode + combine kernels) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def run_decode(case: W.DecodeCase, out_dtype=torch.float32):
    import exact_attention_158_b200 as fa
    inp = W.make_decode(case, device="cuda")
    o, lse = fa.fa_decode_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                inp["seq_lens"], scale=case.scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    o_ref, lse_ref = orc.decode_paged(W.bf16_bits(inp["q"]), W.bf16_bits(inp["k_pool"]),
                                      W.bf16_bits(inp["v_pool"]), inp["block_table"].cpu().numpy(),
                                      inp["seq_lens"].cpu().numpy(), case.scale)
    parity.assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, case.name,
                        out_bf16=out_dtype == torch.bfloat16)
    return inp, o, lse


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_decode_config(out_dtype):
    # 64 sequences, H=32, d=128, context lengths uniform in [512, 8192], 16-token blocks
    run_decode(W.DecodeCase("decode"), out_dtype)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("lens", [[1], [15, 16, 17], [1, 511, 512, 513, 1024, 3000]])
def test_decode_edge_lengths(d, lens):
    run_decode(W.DecodeCase(f"edge_d{d}", S=len(lens), H=4, d=d, lens=lens))


def test_decode_equals_last_causal_row():
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("x", S=3, H=4, d=128, lens=[700, 129, 2048])
    inp = W.make_decode(case, device="cuda")
    o_dec, lse_dec = fa.fa_decode_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                        inp["seq_lens"], out_dtype=torch.float32)
    table = inp["block_table"].cpu()
    for s, L in enumerate(case.lens):
        pages = table[s, : -(-L // 16)].long().cuda()
        k = inp["k_pool"][pages].permute(1, 0, 2, 3).reshape(case.H, -1, case.d)[:, :L]
        v = inp["v_pool"][pages].permute(1, 0, 2, 3).reshape(case.H, -1, case.d)[:, :L]
        q = torch.zeros_like(k)
        q[:, -1] = inp["q"][s]
        o, lse = fa.fa_fwd(q[None].contiguous(), k[None].contiguous(), v[None].contiguous(),
                           causal=True, out_dtype=torch.float32)
        torch.cuda.synchronize()
        d = (o[0, :, -1] - o_dec[s]).abs().max().item()
        assert d <= 1e-2, f"seq {s}: decode vs last causal row {d}"
        assert (lse[0, :, -1] - lse_dec[s]).abs().max().item() <= 1e-3


def test_pool_relocation_is_bitwise_invariant():
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("reloc", S=5, H=4, d=64, lens=[33, 900, 17, 1600, 2])
    inp = W.make_decode(case, device="cuda")
    o1, l1 = fa.fa_decode_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                inp["seq_lens"])
    P = inp["num_blocks"]
    pi = torch.randperm(P, generator=torch.Generator().manual_seed(3)).cuda()
    k2 = torch.empty_like(inp["k_pool"])
    v2 = torch.empty_like(inp["v_pool"])
    k2[pi] = inp["k_pool"]
    v2[pi] = inp["v_pool"]
    t = inp["block_table"].long()
    t2 = torch.where(t >= 0, pi[t.clamp(min=0)], -1).to(torch.int32)
    o2, l2 = fa.fa_decode_paged(inp["q"], k2, v2, t2, inp["seq_lens"])
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_block_id_is_reported_not_read():
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("bad", S=2, H=2, d=128, lens=[40, 40])
    inp = W.make_decode(case, device="cuda")
    table = inp["block_table"].clone()
    table[1, 1] = inp["num_blocks"] + 5  # outside the pool: the kernel must skip it and report
    fa.fa_decode_paged(inp["q"], inp["k_pool"], inp["v_pool"], table, inp["seq_lens"])
    assert fa.device_status() == 1
    assert fa.device_status() == 0  # reading clears it


def test_decode_long_context():
    # one 131072-token context (8192 pages, 256 split chunks) beside short ones
    run_decode(W.DecodeCase("long", S=3, H=4, d=128, lens=[131072, 5, 777]))
