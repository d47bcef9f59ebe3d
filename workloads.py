"""Seeded synthetic inputs for exact attention (shared by the CUDA path's tests/bench and the oracle).

This module only draws numbers and lays them out; it holds none of the attention arithmetic.
Both sides receive the very same bf16 bytes from here.

Generator (counter based, so any element can be drawn independently on any device):

* ``splitmix64(x)``: the published SplitMix64 finaliser (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): add the golden gamma 0x9E3779B97F4A7C15, then
  xor-shift-multiply by 0xBF58476D1CE4E5B9 (shift 30) and 0x94D049BB133111EB (shift 27), xor-shift 31.
* stream key of a tensor: ``key = splitmix64(seed ^ splitmix64(tensor_id))``;
  the raw word of element ``i`` is ``splitmix64(key + i)`` (mod 2^64).
* normals by Box-Muller over pairs (2k, 2k+1): ``u1 = ((w_2k >> 11) + 1) / 2^53`` in (0, 1],
  ``u2 = (w_2k+1 >> 11) / 2^53``; ``z_2k = r cos(2 pi u2)``, ``z_2k+1 = r sin(2 pi u2)`` with
  ``r = sqrt(-2 ln u1)``, evaluated in fp64, rounded to fp32, then to bf16 (round to nearest even).

Tensor ids: Q=1, K=2, V=3, context lengths=4, block-table permutation=5, peaked key rows=6.
Base seed 158.

Workload shapes follow the FlashAttention-2 benchmark grid described on "FlashAttention-2 GPU work
partitioning" (section 4: sequence length 512 to about 16k, head dimension 64 and 128, causal on/off,
16k tokens in total per batch) and the paged KV cache of "LLM study notes" (paged attention: a block
table maps a sequence's logical KV blocks onto scattered physical blocks).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BASE_SEED = 158
TID_Q, TID_K, TID_V, TID_LENS, TID_PERM, TID_PEAKS, TID_DO, TID_TREE = 1, 2, 3, 4, 5, 6, 7, 8
PAGE_SIZE = 16

_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB


def _s64(x: int) -> int:
    """Two's-complement view of a 64-bit word (torch has no uint64 arithmetic)."""
    x &= _M64
    return x - (1 << 64) if x >= (1 << 63) else x


def splitmix64_int(x: int) -> int:
    """SplitMix64 on one Python integer (exact, mod 2^64)."""
    z = (x + _GAMMA) & _M64
    z = ((z ^ (z >> 30)) * _C1) & _M64
    z = ((z ^ (z >> 27)) * _C2) & _M64
    return z ^ (z >> 31)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    # logical right shift of int64 words
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64(x: torch.Tensor) -> torch.Tensor:
    """SplitMix64 on an int64 tensor (wrapping arithmetic), any device."""
    z = x + _s64(_GAMMA)
    z = (z ^ _lsr(z, 30)) * _s64(_C1)
    z = (z ^ _lsr(z, 27)) * _s64(_C2)
    return z ^ _lsr(z, 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return splitmix64_int((seed ^ splitmix64_int(tensor_id)) & _M64)


def raw_words(seed: int, tensor_id: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Raw 64-bit words (as int64) of elements start .. start+count-1 of one stream."""
    key = stream_key(seed, tensor_id)
    idx = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return splitmix64(idx + _s64(key))


def _top53(w: torch.Tensor) -> torch.Tensor:
    return _lsr(w, 11).to(torch.float64)


def normal_bf16(seed: int, tensor_id: int, numel: int, device="cpu", chunk: int = 1 << 26,
                first: int = 0) -> torch.Tensor:
    """``numel`` N(0,1) draws rounded to bf16: elements first .. first+numel-1 of the stream
    (``first`` even, so that Box-Muller pairs line up with the full tensor's)."""
    if first % 2:
        raise ValueError("first must be even")
    out = torch.empty(numel, dtype=torch.bfloat16, device=device)
    two53 = float(1 << 53)
    start = 0
    while start < numel:
        # pairs must start on an even index
        n = min(chunk, numel - start)
        npair = (n + 1) // 2
        w = raw_words(seed, tensor_id, first + start, 2 * npair, device)
        w = w.view(npair, 2)
        u1 = (_top53(w[:, 0]) + 1.0) / two53
        u2 = _top53(w[:, 1]) / two53
        r = torch.sqrt(-2.0 * torch.log(u1))
        ang = (2.0 * math.pi) * u2
        z = torch.stack((r * torch.cos(ang), r * torch.sin(ang)), dim=1).reshape(-1)[:n]
        out[start:start + n] = z.to(torch.float32).to(torch.bfloat16)
        del w, u1, u2, r, ang, z
        start += n
    return out


def uniform_ints(seed: int, tensor_id: int, count: int, lo: int, hi: int, start: int = 0) -> list[int]:
    """``count`` integers in [lo, hi] (inclusive): lo + (word mod (hi - lo + 1)), word unsigned."""
    key = stream_key(seed, tensor_id)
    span = hi - lo + 1
    return [lo + (splitmix64_int((key + start + i) & _M64) % span) for i in range(count)]


def random_permutation(seed: int, tensor_id: int, n: int) -> torch.Tensor:
    """A permutation of 0..n-1: indices sorted by their raw words (ties by index; words are 64-bit)."""
    w = raw_words(seed, tensor_id, 0, n)
    # order by the unsigned value: flip the sign bit so signed order equals unsigned order
    keyed = w ^ _s64(1 << 63)
    return torch.argsort(keyed, stable=True).to(torch.int64)


# --------------------------------------------------------------------------------------------
# prefill workloads
# --------------------------------------------------------------------------------------------

@dataclass
class PrefillCase:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    peaked: bool = False          # 1 % of key rows of every (b, h) scaled by peak_factor
    peak_factor: int = 8          # a power of two, so the scaled bf16 rows are exact
    seed: int = BASE_SEED
    rising: bool = False          # key blocks scaled by rising_factor (x1, then x8, then x64)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """Algorithmic attention FLOPs: 4 B H N^2 d, halved for causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f


def peaked_rows(seed: int, bh: int, N: int) -> list[int]:
    """ceil(N/100) distinct key rows of head ``bh``, by a partial Fisher-Yates shuffle of 0..N-1.

    Draw t (t = 0 .. r-1) of head bh uses word index bh * N + t of the peaks stream.
    """
    r = -(-N // 100)
    idx = list(range(N))
    key = stream_key(seed, TID_PEAKS)
    for t in range(r):
        w = splitmix64_int((key + bh * N + t) & _M64)
        j = t + (w % (N - t))
        idx[t], idx[j] = idx[j], idx[t]
    return sorted(idx[:r])


def rising_factor(pos: int, n: int) -> int:
    """Scale of the key at position ``pos`` of a length-``n`` sequence in the "rising" inputs: its
    128-key block b of nb = ceil(n/128) gets 1 in the first third (3b < nb), 8 in the second
    (3b < 2nb) and 64 in the last.  Powers of two, so the scaled bf16 keys are exact; the row
    maxima of the scores then jump by far more than 2^8 (in log2 units) after the first block."""
    nb = -(-n // 128)
    b = pos // 128
    return 1 if 3 * b < nb else (8 if 3 * b < 2 * nb else 64)


def make_prefill(case: PrefillCase, device="cpu"):
    """Q, K, V as bf16 tensors of shape [B, H, N, d] (contiguous), on ``device``."""
    shape = (case.B, case.H, case.N, case.d)
    numel = case.B * case.H * case.N * case.d
    q = normal_bf16(case.seed, TID_Q, numel, device).view(shape)
    k = normal_bf16(case.seed, TID_K, numel, device).view(shape)
    v = normal_bf16(case.seed, TID_V, numel, device).view(shape)
    if case.peaked:
        kf = k.view(case.B * case.H, case.N, case.d)
        for bh in range(case.B * case.H):
            rows = torch.tensor(peaked_rows(case.seed, bh, case.N), device=device)
            kf[bh, rows] = kf[bh, rows] * case.peak_factor  # power of two: exact in bf16
    if case.rising:
        f = torch.tensor([rising_factor(p, case.N) for p in range(case.N)], dtype=torch.bfloat16,
                         device=device)
        k.mul_(f.view(1, 1, case.N, 1))
    return q, k, v


def make_prefill_heads(case: PrefillCase, heads, device="cpu"):
    """Q, K, V of the listed (b, h) slices only (flat index bh = b * H + h), as bf16 tensors
    [len(heads), N, d]: the same values make_prefill gives those slices, without drawing the rest."""
    N, d = case.N, case.d
    out = []
    for tid in (TID_Q, TID_K, TID_V):
        t = torch.stack([normal_bf16(case.seed, tid, N * d, device, first=bh * N * d).view(N, d)
                         for bh in heads])
        out.append(t)
    q, k, v = out
    for i, bh in enumerate(heads):
        if case.peaked:
            rows = torch.tensor(peaked_rows(case.seed, bh, N), device=device)
            k[i, rows] = k[i, rows] * case.peak_factor
    if case.rising:
        f = torch.tensor([rising_factor(p, N) for p in range(N)], dtype=torch.bfloat16,
                         device=device)
        k.mul_(f.view(1, N, 1))
    return q, k, v


def tiny_cases():
    return [PrefillCase("tiny", 1, 1, 256, 64, c) for c in (False, True)]


def prefill_cases():
    return [PrefillCase("prefill", 8, 16, 2048, 128, c) for c in (False, True)]


def sweep_cases(d: int):
    out = []
    for N in (512, 1024, 2048, 4096, 8192, 16384):
        H = 2048 // d
        for c in (False, True):
            out.append(PrefillCase(f"sweep_d{d}", 16384 // N, H, N, d, c, peaked=(d == 64)))
    return out


# --------------------------------------------------------------------------------------------
# paged decode workload
# --------------------------------------------------------------------------------------------

POISON_K = 8192.0       # a large finite bf16 value written into unused page slots of K
POISON_V = 1.0e4        # +- this into unused page slots of V (bf16 rounds it to 9984)


@dataclass
class DecodeCase:
    name: str
    S: int = 64                 # sequences, query length 1
    H: int = 32
    d: int = 128
    len_lo: int = 512
    len_hi: int = 8192
    seed: int = BASE_SEED
    lens: list = field(default=None)  # optional explicit context lengths
    rising: bool = False        # keys scaled by rising_factor of their position in the sequence

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def seq_lens(self) -> list[int]:
        if self.lens is not None:
            return list(self.lens)
        return uniform_ints(self.seed, TID_LENS, self.S, self.len_lo, self.len_hi)


def make_dout(case: PrefillCase, device="cpu"):
    """The incoming gradient dO for the backward pass: bf16 [B, H, N, d], i.i.d. N(0, 1)."""
    shape = (case.B, case.H, case.N, case.d)
    return normal_bf16(case.seed, TID_DO, case.B * case.H * case.N * case.d, device).view(shape)


def make_decode(case: DecodeCase, device="cpu"):
    """Paged decode inputs.

    Returns dict with q [S,H,d] bf16, k_pool/v_pool [P,H,16,d] bf16, block_table [S,max_blocks] int32
    (unused entries -1), seq_lens [S] int32, num_blocks P, and max_blocks.
    The pool holds exactly sum_s ceil(L_s/16) pages; the logical pages of all sequences, in order,
    are mapped onto a seeded random permutation of the pool.  Slots past L_s in a sequence's last
    page are poisoned (K = POISON_K, V = +-POISON_V) so any read of them shows up in the output.
    """
    lens = case.seq_lens()
    nblk = [-(-L // PAGE_SIZE) for L in lens]
    P = sum(nblk)
    maxb = max(nblk)
    perm = random_permutation(case.seed, TID_PERM, P)
    table = torch.full((case.S, maxb), -1, dtype=torch.int32)
    off = 0
    for s in range(case.S):
        table[s, :nblk[s]] = perm[off:off + nblk[s]].to(torch.int32)
        off += nblk[s]
    page_elems = case.H * PAGE_SIZE * case.d
    q = normal_bf16(case.seed, TID_Q, case.S * case.H * case.d, device).view(case.S, case.H, case.d)
    k_pool = normal_bf16(case.seed, TID_K, P * page_elems, device).view(P, case.H, PAGE_SIZE, case.d)
    v_pool = normal_bf16(case.seed, TID_V, P * page_elems, device).view(P, case.H, PAGE_SIZE, case.d)
    if case.rising:
        # 128-key blocks start on page boundaries, so one factor covers a whole page
        for s in range(case.S):
            for pg in range(nblk[s]):
                f = rising_factor(pg * PAGE_SIZE, lens[s])
                if f != 1:
                    blk = int(table[s, pg])
                    k_pool[blk] = k_pool[blk] * f
    for s in range(case.S):
        tail = lens[s] % PAGE_SIZE
        if tail:
            last = int(table[s, nblk[s] - 1])
            k_pool[last, :, tail:, :] = POISON_K
            sign = torch.where(torch.arange(case.d, device=device) % 2 == 0, 1.0, -1.0)
            v_pool[last, :, tail:, :] = (POISON_V * sign).to(torch.bfloat16)
    seq_lens = torch.tensor(lens, dtype=torch.int32)
    return dict(q=q, k_pool=k_pool, v_pool=v_pool, block_table=table.to(device),
                seq_lens=seq_lens.to(device), num_blocks=P, max_blocks=maxb, lens=lens)


def make_paged_prefill(case: DecodeCase, Lq: int, device="cpu"):
    """Chunked prefill over a paged cache: the decode case's pool, table and lengths (each length
    must be >= Lq), plus q [S,H,Lq,d] for the last Lq positions of every sequence."""
    inp = make_decode(case, device)
    if min(inp["lens"]) < Lq:
        raise ValueError("every context must hold the Lq chunk")
    inp["q"] = normal_bf16(case.seed, TID_Q, case.S * case.H * Lq * case.d, device).view(
        case.S, case.H, Lq, case.d)
    inp["Lq"] = Lq
    return inp


def paged_prefill_flops(lens, H: int, d: int, Lq: int, causal: bool) -> int:
    """Matmul FLOPs of a chunked prefill: 4 d per visible (query, key) pair (Q K^T and P V).  The
    chunk's query t of a length-L context sees L - Lq + t + 1 keys causally, else all L."""
    pairs = 0
    for L in lens:
        pairs += Lq * (L - Lq) + Lq * (Lq + 1) // 2 if causal else Lq * L
    return 4 * d * H * pairs


def random_tree_parents(seed: int, S: int, T: int, shape: str = "random") -> list[list[int]]:
    """Draft-token trees, one per sequence, as parent lists in topological order: node t's parent
    is -1 (it follows the context directly) or an earlier node.  shape: "random" (parent of t
    uniform over -1 .. t-1, seeded), "chain" (t - 1), "star" (all -1)."""
    trees = []
    for s in range(S):
        if shape == "chain":
            trees.append([t - 1 for t in range(T)])
        elif shape == "star":
            trees.append([-1] * T)
        else:
            draws = uniform_ints(seed, TID_TREE, T, 0, 1 << 30, start=s * T)
            trees.append([(w % (t + 1)) - 1 for t, w in enumerate(draws)])
    return trees


def tree_visibility(parents: list[int]) -> list[int]:
    """Bit u of entry t is set when node u is node t itself or one of its ancestors: the draft
    tokens on the path from the context to t (the sequence node t continues)."""
    bits = []
    for t, par in enumerate(parents):
        if not -1 <= par < t:
            raise ValueError("parents must point to an earlier node or -1")
        bits.append((1 << t) | (bits[par] if par >= 0 else 0))
    return bits


def make_tree_verify(case: "DecodeCase", T: int, shape: str = "random", device="cpu"):
    """Tree verification over a paged cache: the decode case's pool, table and lengths (each length
    >= T, the last T cached tokens being the tree's nodes in topological order), q [S,H,T,d] for the
    nodes, and the visibility masks as int64 [S, T] (the bit pattern of uint64; T <= 64)."""
    if not 1 <= T <= 64:
        raise ValueError("tree size must be in [1, 64]")
    inp = make_paged_prefill(case, T, device)
    parents = random_tree_parents(case.seed, case.S, T, shape)
    masks = [tree_visibility(p) for p in parents]
    signed = [[m - (1 << 64) if m >= 1 << 63 else m for m in row] for row in masks]
    inp["parents"] = parents
    inp["tree_mask"] = torch.tensor(signed, dtype=torch.int64).to(device)
    inp["T"] = T
    return inp


def tree_verify_flops(lens, masks, H: int, d: int) -> int:
    """Matmul FLOPs of tree verification: 4 d per visible (node, key) pair; node t of a length-L
    context sees the L - T context tokens and the nodes set in its mask."""
    pairs = 0
    for L, row in zip(lens, masks):
        T = len(row)
        pairs += sum((L - T) + bin(m & ((1 << 64) - 1)).count("1") for m in row)
    return 4 * d * H * pairs


def tree_verify_bytes(lens, H: int, d: int, T: int) -> int:
    """Algorithmic bytes of one tree verification: K and V of every cached token (bf16), the
    nodes' q and o (bf16), their masks (uint64), the used block-table entries and the lengths."""
    S = len(lens)
    pages = sum(-(-L // PAGE_SIZE) for L in lens)
    return 2 * H * d * 2 * sum(lens) + 2 * S * H * T * d * 2 + 8 * S * T + 4 * pages + 4 * S


def decode_bytes(lens, H: int, d: int, max_blocks: int) -> int:
    """Algorithmic bytes of one paged decode pass: K and V of every context token (bf16), q and o
    (bf16), the block-table entries actually used (int32) and the lengths (int32)."""
    S = len(lens)
    tokens = sum(lens)
    pages = sum(-(-L // PAGE_SIZE) for L in lens)
    return 2 * H * d * 2 * tokens + 2 * S * H * d * 2 + 4 * pages + 4 * S


def bf16_bits(t: torch.Tensor):
    """The raw 16-bit patterns of a bf16 tensor as a contiguous numpy uint16 array (CPU copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
