import pytest
"""The seeded input generator and the workload shapes (no GPU)."""
import json
import math
import os

import numpy as np
import torch

import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_first_output():
    # SplitMix64 seeded with 0: the first output of the published generator
    assert W.splitmix64_int(0) == 0xE220A8397B1DCDAF


def test_splitmix64_tensor_matches_integer_version():
    xs = [0, 1, 2, 12345, 2**63 - 1, 2**63, 2**64 - 1, 0x9E3779B97F4A7C15]
    t = W.splitmix64(torch.tensor([W._s64(x) for x in xs], dtype=torch.int64))
    got = [int(v) & W._M64 for v in t.tolist()]
    assert got == [W.splitmix64_int(x) for x in xs]


def test_normals_chunk_invariant_and_standard():
    a = W.normal_bf16(158, W.TID_Q, 100_003)
    b = W.normal_bf16(158, W.TID_Q, 100_003, chunk=4096)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    x = a.float()
    assert abs(float(x.mean())) < 0.02 and abs(float(x.std()) - 1) < 0.02
    c = W.normal_bf16(158, W.TID_K, 100_003)
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_benchmark_grid_matches_page():
    g = json.load(open(os.path.join(GOLDEN, "fa2_benchmark_grid.json")))
    for d in g["head_dims"]:
        cases = W.sweep_cases(d)
        assert sorted({c.N for c in cases}) == g["seqlens"]
        assert {c.causal for c in cases} == set(g["causal"])
        for c in cases:
            assert c.B * c.N == g["total_tokens"]
            assert c.H * c.d == g["hidden"]
            assert c.peaked == (d == 64)


def test_flop_count():
    c = W.PrefillCase("x", 8, 16, 2048, 128, False)
    assert c.flops == 4 * 8 * 16 * 2048 ** 2 * 128
    assert W.PrefillCase("x", 8, 16, 2048, 128, True).flops == c.flops / 2


def test_peaked_rows():
    case = W.PrefillCase("p", 2, 2, 300, 64, False, peaked=True)
    q, k, v = W.make_prefill(case)
    plain = W.make_prefill(W.PrefillCase("p", 2, 2, 300, 64, False))[1]
    kf, pf = k.view(4, 300, 64).float(), plain.view(4, 300, 64).float()
    for bh in range(4):
        rows = W.peaked_rows(case.seed, bh, 300)
        assert len(rows) == len(set(rows)) == math.ceil(300 / 100)
        scaled = [r for r in range(300) if not torch.equal(kf[bh, r], pf[bh, r])]
        assert scaled == rows
        assert torch.equal(kf[bh, rows], pf[bh, rows] * 8)


def test_paged_layout_and_waste():
    g = json.load(open(os.path.join(GOLDEN, "paged_block_example.json")))
    # the page's example: block size 4 wastes at most 3 slots
    for L in range(1, 50):
        assert -(-L // g["block_size"]) * g["block_size"] - L <= g["max_wasted_slots"]
    case = W.DecodeCase("t", S=5, H=2, d=16, lens=[1, 16, 17, 33, 100])
    inp = W.make_decode(case)
    table = inp["block_table"]
    used = []
    for s, L in enumerate(case.lens):
        nb = -(-L // W.PAGE_SIZE)
        assert nb * W.PAGE_SIZE - L <= W.PAGE_SIZE - 1
        assert bool((table[s, :nb] >= 0).all()) and bool((table[s, nb:] == -1).all())
        used += table[s, :nb].tolist()
    assert sorted(used) == list(range(inp["num_blocks"]))
    # poisoned tail slots
    s = 0
    last = int(table[s, 0])
    assert bool((inp["k_pool"][last, :, 1:, :].float() == W.POISON_K).all())


def test_decode_lengths_in_range():
    lens = W.DecodeCase("d").seq_lens()
    assert len(lens) == 64 and min(lens) >= 512 and max(lens) <= 8192
    assert len(set(lens)) > 50


def test_paged_prefill_flops_counts_visible_pairs():
    lens, Lq, H, d = [5, 9, 20], 4, 3, 8
    for causal in (True, False):
        pairs = sum(1 for L in lens for t in range(Lq) for key in range(L)
                    if not causal or key <= L - Lq + t)
        assert W.paged_prefill_flops(lens, H, d, Lq, causal) == 4 * d * H * pairs


def test_tree_visibility_is_the_ancestor_set():
    for shape in ("random", "star", "chain"):
        for parents in W.random_tree_parents(5, 3, 40, shape):
            bits = W.tree_visibility(parents)
            for t in range(40):
                anc, u = set(), t
                while u >= 0:
                    anc.add(u)
                    u = parents[u]
                assert {u for u in range(40) if bits[t] >> u & 1} == anc
    with pytest.raises(ValueError):
        W.tree_visibility([0])


def test_tree_verify_flops_counts_visible_pairs():
    parents = [[-1, 0, 0, 1], [-1, -1, 1, 2]]
    masks = [W.tree_visibility(p) for p in parents]
    lens = [10, 4]
    pairs = 0
    for L, p in zip(lens, parents):
        for t in range(4):
            anc, u = 0, t
            while u >= 0:
                anc, u = anc + 1, p[u]
            pairs += (L - 4) + anc
    assert W.tree_verify_flops(lens, masks, 3, 8) == 4 * 8 * 3 * pairs


def test_head_subset_generator_matches_full_tensors():
    # the bench's per-point oracle samples draw only a few (b, h) slices; they must be the very
    # slices the full generator produces, peaked and rising variants included
    for case in (W.PrefillCase("h", 2, 3, 300, 64, False, peaked=True),
                 W.PrefillCase("h", 1, 2, 1000, 128, True, rising=True)):
        full = W.make_prefill(case)
        heads = [0, case.B * case.H - 1]
        part = W.make_prefill_heads(case, heads)
        for a, b in zip(full, part):
            assert torch.equal(a.reshape(-1, case.N, case.d)[heads], b)
