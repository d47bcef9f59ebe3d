"""fa_tree_attention (draft-tree verification over the paged cache) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def run_tree(case: W.DecodeCase, T: int, shape="random", out_dtype=torch.float32, mask=None):
    import exact_attention_158_b200 as fa
    inp = W.make_tree_verify(case, T, shape, device="cuda")
    tm = inp["tree_mask"] if mask is None else mask
    o, lse = fa.fa_tree_attention(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                  inp["seq_lens"], tm, scale=case.scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    o_ref, lse_ref = orc.tree_attention(W.bf16_bits(inp["q"]), W.bf16_bits(inp["k_pool"]),
                                        W.bf16_bits(inp["v_pool"]), inp["block_table"].cpu().numpy(),
                                        inp["seq_lens"].cpu().numpy(), tm.cpu().numpy(), case.scale)
    return inp, o, lse, o_ref, lse_ref


# contexts of 0 .. 2000 tokens before the tree (lengths include the T nodes), ragged against the
# 16-token page and the 128-key tile
CONTEXTS = [0, 1, 100, 127, 128, 300, 2000]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 7, 33, 64])
def test_tree_random(d, T):
    case = W.DecodeCase(f"tree_d{d}", S=len(CONTEXTS), H=2, d=d, lens=[c + T for c in CONTEXTS])
    _, o, lse, o_ref, lse_ref = run_tree(case, T)
    parity.assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref,
                        f"tree d={d} T={T}")


@pytest.mark.parametrize("shape", ["chain", "star"])
def test_tree_shapes(shape):
    case = W.DecodeCase("tree_shape", S=3, H=2, d=128, lens=[64, 200, 1064])
    _, o, lse, o_ref, lse_ref = run_tree(case, 64, shape)
    parity.assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"tree {shape}")


@pytest.mark.parametrize("d", [64, 128])
def test_tree_bf16_out(d):
    case = W.DecodeCase(f"tree_bf16_d{d}", S=4, H=4, d=d, lens=[96, 300, 1000, 50])
    _, o, lse, o_ref, lse_ref = run_tree(case, 40, out_dtype=torch.bfloat16)
    parity.assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "tree bf16",
                        out_bf16=True)


def test_tree_workload():
    # verification shape: long contexts, a 64-node random tree per sequence
    case = W.DecodeCase("tree_work", S=6, H=8, d=128, len_lo=1024, len_hi=4096)
    _, o, lse, o_ref, lse_ref = run_tree(case, 64)
    parity.assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "tree workload")


def test_chain_tree_equals_causal_chunk():
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("tree_chain", S=3, H=2, d=64, lens=[70, 500, 129])
    inp, o, lse, _, _ = run_tree(case, 50, "chain")
    oc, lc = fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                 inp["seq_lens"], causal=True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o, oc) and torch.equal(lse, lc)


def test_node_that_sees_nothing():
    # no context, and node 5's mask cleared: O = 0, LSE = -inf; the other rows are unaffected
    case = W.DecodeCase("tree_empty", S=1, H=2, d=128, lens=[16])
    inp = W.make_tree_verify(case, 16, "random", device="cuda")
    mask = inp["tree_mask"].clone()
    mask[0, 5] = 0
    _, o, lse, o_ref, lse_ref = run_tree(case, 16, mask=mask)
    assert torch.all(o[0, :, 5] == 0) and torch.all(torch.isneginf(lse[0, :, 5]))
    keep = [t for t in range(16) if t != 5]
    parity.assert_close(o[0][:, keep].float().cpu().numpy(), lse[0][:, keep].cpu().numpy(),
                        o_ref[0][:, keep], lse_ref[0][:, keep], "tree empty row, other rows")
