"""fa_prefill_paged (chunked prefill over a paged KV cache) against the fp64 oracle, plus its
consistency with the decode and dense entry points."""
import pytest
import torch

import workloads as W
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def run_paged(case: W.DecodeCase, Lq: int, causal: bool, out_dtype=torch.float32):
    import exact_attention_158_b200 as fa
    inp = W.make_paged_prefill(case, Lq, device="cuda")
    o, lse = fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                 inp["seq_lens"], causal=causal, scale=case.scale,
                                 out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    o_ref, lse_ref = orc.prefill_paged(W.bf16_bits(inp["q"]), W.bf16_bits(inp["k_pool"]),
                                       W.bf16_bits(inp["v_pool"]), inp["block_table"].cpu().numpy(),
                                       inp["seq_lens"].cpu().numpy(), causal, case.scale)
    parity.assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref,
                        f"{case.name} Lq={Lq} causal={causal}", out_bf16=out_dtype == torch.bfloat16)
    return inp, o, lse


# Lengths that are not multiples of the 16-token page nor of the 128-key tile, chunks that end
# inside a tile, span several tiles, or are the whole context.
LENS = [300, 129, 1000, 517, 2048]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("Lq", [1, 7, 128, 129])
def test_paged_prefill_chunks(d, causal, Lq):
    run_paged(W.DecodeCase(f"pp_d{d}", S=len(LENS), H=3, d=d, lens=LENS), Lq, causal)


@pytest.mark.parametrize("d", [64, 128])
def test_paged_prefill_whole_context_chunk(d):
    # Lq equal to the shortest context: that sequence's chunk is its whole context
    lens = [257, 700, 1500]
    run_paged(W.DecodeCase(f"pp_whole_d{d}", S=3, H=2, d=d, lens=lens), 257, True)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Lq", [100, 300])
@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
def test_paged_prefill_bf16_out(causal, Lq, d):
    # bf16 O leaves through tensor stores of 32-row boxes, clipped at row Lq
    run_paged(W.DecodeCase(f"pp_bf16_d{d}", S=4, H=4, d=d, lens=[600, 333, 1024, 329]), Lq, causal,
              out_dtype=torch.bfloat16)


def test_paged_prefill_chunked_workload():
    # chunked-prefill shape: several sequences with long cached contexts, 512-token chunks
    case = W.DecodeCase("pp_chunked", S=4, H=8, d=128, len_lo=1024, len_hi=4096)
    run_paged(case, 512, True)


def test_chunk_of_one_equals_decode():
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("pp_dec", S=4, H=4, d=128, lens=[1, 17, 640, 2000])
    inp = W.make_paged_prefill(case, 1, device="cuda")
    o, lse = fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                 inp["seq_lens"], causal=True, out_dtype=torch.float32)
    o_d, lse_d = fa.fa_decode_paged(inp["q"][:, :, 0].contiguous(), inp["k_pool"], inp["v_pool"],
                                    inp["block_table"], inp["seq_lens"], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (o[:, :, 0] - o_d).abs().max().item() <= 1e-2
    assert (lse[:, :, 0] - lse_d).abs().max().item() <= 1e-3


def test_whole_context_equals_dense_causal():
    # one sequence whose chunk is its whole context is the dense causal problem
    import exact_attention_158_b200 as fa
    L, H, d = 777, 4, 64
    case = W.DecodeCase("pp_dense", S=1, H=H, d=d, lens=[L])
    inp = W.make_paged_prefill(case, L, device="cuda")
    o, lse = fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                 inp["seq_lens"], causal=True, out_dtype=torch.float32)
    pages = inp["block_table"][0, : -(-L // 16)].long()
    k = inp["k_pool"][pages].permute(1, 0, 2, 3).reshape(H, -1, d)[:, :L]
    v = inp["v_pool"][pages].permute(1, 0, 2, 3).reshape(H, -1, d)[:, :L]
    o_f, lse_f = fa.fa_fwd(inp["q"], k[None].contiguous(), v[None].contiguous(), causal=True,
                           out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (o - o_f).abs().max().item() <= 1e-2
    assert (lse - lse_f).abs().max().item() <= 1e-3


def test_pool_relocation_is_bitwise_invariant():
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("pp_reloc", S=3, H=2, d=128, lens=[300, 45, 1111])
    inp = W.make_paged_prefill(case, 40, device="cuda")
    args = dict(causal=True, out_dtype=torch.float32)
    o1, l1 = fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                 inp["seq_lens"], **args)
    P = inp["num_blocks"]
    pi = torch.randperm(P, generator=torch.Generator().manual_seed(5)).cuda()
    k2 = torch.empty_like(inp["k_pool"])
    v2 = torch.empty_like(inp["v_pool"])
    k2[pi] = inp["k_pool"]
    v2[pi] = inp["v_pool"]
    t = inp["block_table"].long()
    t2 = torch.where(t >= 0, pi[t.clamp(min=0)], -1).to(torch.int32)
    o2, l2 = fa.fa_prefill_paged(inp["q"], k2, v2, t2, inp["seq_lens"], **args)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bad", ["past_pool", "negative"])
def test_bad_block_id_is_reported_not_read(d, bad):
    # d = 128 gathers whole pages through a map indexed block * H + head: an entry past the pool
    # or negative must still land out of range (zeros), never on another head's or block's page
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("pp_bad", S=2, H=2, d=d, lens=[200, 64])
    inp = W.make_paged_prefill(case, 16, device="cuda")
    table = inp["block_table"].clone()
    table[0, 3] = inp["num_blocks"] + 1000 if bad == "past_pool" else -7
    o, lse = fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], table, inp["seq_lens"],
                                 out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.device_status() == 1  # FA_ERR_INVALID_ARG
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    # the error word is cleared by the read; a good call afterwards reports nothing
    fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                        inp["seq_lens"])
    torch.cuda.synchronize()
    assert fa.device_status() == 0


def test_length_shorter_than_chunk_is_reported():
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("pp_short", S=2, H=2, d=128, lens=[300, 200])
    inp = W.make_paged_prefill(case, 64, device="cuda")
    lens = inp["seq_lens"].clone()
    lens[1] = 10  # fewer cached tokens than the chunk claims
    fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"], lens)
    torch.cuda.synchronize()
    assert fa.device_status() == 1  # FA_ERR_INVALID_ARG
