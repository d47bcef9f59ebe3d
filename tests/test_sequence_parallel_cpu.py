"""Host logic of the sequence-sharded forward on CPU with gloo (world size 2 and 3): each rank
holds one key range, computes the partials of all queries over it, the ranks all-gather them and
merge.  The partial and merge steps are the fp64 oracle's here (the GPU path runs the kernels), so
the check is that the ranges, the exchange and the merge order reproduce plain attention."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import workloads as W
    from oracle import oracle as orc
    from exact_attention_158_b200 import sequence_parallel as sp

    case = W.PrefillCase("sp", 1, 2, 100, 16, causal)
    q, k, v = W.make_prefill(case)
    a, b = sp.key_ranges(case.N, world)[rank]

    def partial(q_, k_, v_, k_pos0, causal_, scale_):
        o, lse = orc.attention_keyrange(W.bf16_bits(q_), W.bf16_bits(k_), W.bf16_bits(v_), 0,
                                        k_pos0, causal_, scale_)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(o_parts, lse_parts, out_dtype):
        o, lse = orc.merge_partials(o_parts.numpy(), lse_parts.numpy())
        return torch.from_numpy(o), torch.from_numpy(lse)

    o, lse = sp.sequence_parallel_attention(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(),
                                            a, causal=causal, scale=case.scale, partial=partial,
                                            merge=merge)
    ref_o, ref_l = orc.attention(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), causal, case.scale)
    out[rank] = (float(np.abs(o.numpy() - ref_o).max()), float(np.abs(lse.numpy() - ref_l).max()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_sharded_keys_merge_to_plain_attention(world, causal):
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, causal, out), nprocs=world, join=True)
    for rank in range(world):
        do, dl = out[rank]
        assert do < 1e-12 and dl < 1e-12, (rank, do, dl)


def test_key_ranges_tile_the_sequence():
    sys.path.insert(0, ROOT)
    from exact_attention_158_b200 import sequence_parallel as sp
    for N, world in ((100, 3), (8, 8), (1000, 7)):
        r = sp.key_ranges(N, world)
        assert r[0][0] == 0 and r[-1][1] == N
        assert all(a1 == b0 for (_, a1), (b0, _) in zip(r, r[1:]))
        sizes = [b - a for a, b in r]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        sp.key_ranges(3, 4)
