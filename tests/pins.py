"""Pins that tie the fp64 oracle to what the pages and the mathematics fix, independently of the
oracle's own code.  Each pin takes an ``OracleLib`` and raises AssertionError when it does not hold,
so the same checks run against the committed oracle (test_oracle_pins.py) and against builds of it
with a planted mistake (test_oracle_mutants.py), which must each fail at least one pin.

The facts used:
* softmax rows are weights that sum to one ("FlashAttention-2 GPU work partitioning", section 2);
* attention is softmax(Q K^T * scale) V with scale = 1 / sqrt(d_k) ("LLM study notes",
  self-attention steps), so: equal scores give the mean of V; one key gives that key's value;
  a dominant score selects its value row; two keys reduce to the logistic function; a constant
  added to a score row changes nothing but the log-sum-exp; the result is equivariant under
  permutations and linear in V;
* the causal mask shows query i only keys 0..i ("FlashAttention-2 GPU work partitioning", section 4);
* the tiled algorithm of "Flash Attention" (myungum), section 2, computes exact attention, so any
  block sizes give the plain result;
* a paged KV cache is only a relocation of logically contiguous rows ("LLM study notes", paged
  attention);
* a sequence's keys can be split into ranges whose partial results merge with the tiled
  algorithm's rescaling rule ("FlashAttention-2 GPU work partitioning", section 3; "Flash
  Attention" (myungum), section 2);
* a draft-token tree is verified in one pass, each node continuing the context along its path
  ("LLM study notes", speculative decoding), so a node sees its ancestors and itself;
* the backward pass returns the gradients of sum(dO * O) with respect to Q, K and V (the pages
  describe it in prose only: "Paged vs Flash attention", training; "Flash Attention" (myungum),
  section 1, recomputation), so it must agree with central finite differences of the forward
  definition and with torch.autograd through torch.softmax in fp64, and obey the closed forms that
  follow from rows of P summing to one and from the shift invariance of the softmax.
Reference values are formed with numpy/scipy from the widened inputs, never from the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.special as sps
import torch

import workloads as W


def bf16(x) -> np.ndarray:
    """Round to bf16 and return the raw bits (uint16)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def widen(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rnd(shape, seed, tid=W.TID_Q) -> np.ndarray:
    n = int(np.prod(shape))
    return W.bf16_bits(W.normal_bf16(seed, tid, n)).reshape(shape)


def close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert np.all(np.isfinite(a)) and err <= tol, f"{what}: max err {err} > {tol}"


# ------------------------------------------------------------------------------------------------

def pin_uniform_scores(orc):
    """Q = 0: every visible key gets the same weight, so O_i = mean of the visible V rows and
    LSE_i = ln |A_i| (ln N, or ln(i+1) when causal)."""
    N, d = 37, 16
    q = bf16(np.zeros((N, d)))
    k = rnd((N, d), 1, W.TID_K)
    v = rnd((N, d), 1, W.TID_V)
    V = widen(v)
    for causal in (False, True):
        o, lse = orc.attention(q, k, v, causal, 0.25)
        for i in range(N):
            n = i + 1 if causal else N
            close(o[i], V[:n].mean(axis=0), 1e-13, f"uniform O row {i} causal={causal}")
            close(lse[i], math.log(n), 1e-13, f"uniform LSE row {i} causal={causal}")


def pin_single_key(orc):
    """N = 1: O = V and LSE = scale * q.k; and causal row 0 (only key 0 visible) for any N."""
    d = 24
    q = rnd((1, d), 2)
    k = rnd((1, d), 2, W.TID_K)
    v = rnd((1, d), 2, W.TID_V)
    scale = 0.3
    for causal in (False, True):
        o, lse = orc.attention(q, k, v, causal, scale)
        close(o[0], widen(v)[0], 1e-15, "N=1 O")
        close(lse[0], scale * float(widen(q)[0] @ widen(k)[0]), 1e-12, "N=1 LSE")
    N = 19
    q = rnd((N, d), 3)
    k = rnd((N, d), 3, W.TID_K)
    v = rnd((N, d), 3, W.TID_V)
    o, lse = orc.attention(q, k, v, True, scale)
    close(o[0], widen(v)[0], 1e-15, "causal row 0 O")
    close(lse[0], scale * float(widen(q)[0] @ widen(k)[0]), 1e-12, "causal row 0 LSE")


def pin_dominant_score(orc):
    """Orthogonal keys c e_j and queries c e_t: the score gap scale*c^2 (> 60) makes the softmax
    one-hot, so O_t = V_t within exp(-60) and LSE_t = scale c^2 (+ a term below 1e-25)."""
    N = d = 8
    c = 32.0
    scale = 1.0 / math.sqrt(d)
    k = bf16(c * np.eye(N, d))
    v = rnd((N, d), 4, W.TID_V)
    perm = np.array([3, 0, 7, 5, 1, 6, 2, 4])
    q = bf16(c * np.eye(N, d)[perm])
    o, lse = orc.attention(q, k, v, False, scale)
    for i in range(N):
        close(o[i], widen(v)[perm[i]], 1e-20 + 1e-12, f"one-hot O row {i}")
        close(lse[i], scale * c * c, 1e-12, f"one-hot LSE row {i}")


def pin_two_keys_logistic(orc):
    """N = 2 reduces to the logistic function: row i gets weight sigma(s_i0 - s_i1) on v_0 and
    sigma(s_i1 - s_i0) on v_1; LSE = max + log1p(exp(-|s_0 - s_1|)).  The causal row 0 sees v_0."""
    d = 32
    q = rnd((2, d), 5)
    k = rnd((2, d), 5, W.TID_K)
    v = rnd((2, d), 5, W.TID_V)
    scale = 0.2
    Q, K, V = widen(q), widen(k), widen(v)
    s = scale * (Q @ K.T)
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    o, lse = orc.attention(q, k, v, False, scale)
    for i in range(2):
        a = sig(s[i, 0] - s[i, 1])
        close(o[i], a * V[0] + (1 - a) * V[1], 1e-13, f"logistic O row {i}")
        close(lse[i], max(s[i]) + math.log1p(math.exp(-abs(s[i, 0] - s[i, 1]))), 1e-13,
              f"logistic LSE row {i}")
    o, lse = orc.attention(q, k, v, True, scale)
    a = sig(s[1, 0] - s[1, 1])
    close(o[1], a * V[0] + (1 - a) * V[1], 1e-13, "logistic causal O row 1")
    close(o[0], V[0], 1e-15, "logistic causal O row 0")


def pin_shift_invariance(orc):
    """K' = K + 1 u^T adds scale*(q_i . u) to every score of row i: O is unchanged and LSE moves by
    that amount.  Small integers keep K' exact in bf16."""
    rng = np.random.default_rng(6)
    N, d = 23, 8
    Q = rng.integers(-3, 4, (N, d)).astype(np.float64)
    K = rng.integers(-3, 4, (N, d)).astype(np.float64)
    V = rng.integers(-5, 6, (N, d)).astype(np.float64)
    u = rng.integers(-2, 3, (d,)).astype(np.float64)
    scale = 0.125
    for causal in (False, True):
        o1, l1 = orc.attention(bf16(Q), bf16(K), bf16(V), causal, scale)
        o2, l2 = orc.attention(bf16(Q), bf16(K + u[None, :]), bf16(V), causal, scale)
        close(o2, o1, 1e-12, f"shift O causal={causal}")
        close(l2, l1 + scale * (Q @ u), 1e-12, f"shift LSE causal={causal}")


def pin_rows_sum_to_one(orc):
    """Every row of P sums to 1 and masked entries are 0; P matches scipy's softmax of Q K^T*scale."""
    N, d = 64, 16
    q = rnd((N, d), 7)
    k = rnd((N, d), 7, W.TID_K)
    scale = 0.25
    S = scale * (widen(q) @ widen(k).T)
    for causal in (False, True):
        P = orc.probs(q, k, causal, scale)
        close(P.sum(axis=1), np.ones(N), 1e-14, f"row sums causal={causal}")
        if causal:
            assert np.all(P[np.triu_indices(N, 1)] == 0.0), "masked entries of P are not zero"
            S = S.copy()
            S[np.triu_indices(N, 1)] = -np.inf
        close(P, sps.softmax(S, axis=1), 1e-14, f"P vs scipy softmax causal={causal}")


def pin_library_softmax(orc):
    """O = softmax(S) V and LSE = logsumexp(S) formed with numpy/scipy on the widened inputs."""
    B_H, N, d = 3, 41, 16
    q = rnd((B_H, N, d), 8)
    k = rnd((B_H, N, d), 8, W.TID_K)
    v = rnd((B_H, N, d), 8, W.TID_V)
    scale = 1 / 4
    Q, K, V = widen(q), widen(k), widen(v)
    for causal in (False, True):
        o, lse = orc.attention(q, k, v, causal, scale)
        for bh in range(B_H):
            S = scale * Q[bh] @ K[bh].T
            if causal:
                S[np.triu_indices(N, 1)] = -np.inf
            close(o[bh], sps.softmax(S, axis=1) @ V[bh], 1e-13, f"scipy O causal={causal}")
            close(lse[bh], sps.logsumexp(S, axis=1), 1e-13, f"scipy LSE causal={causal}")


def pin_permutation(orc):
    """Non-causal: permuting K and V rows together leaves O unchanged; permuting Q rows permutes O."""
    N, d = 29, 8
    q = rnd((N, d), 9)
    k = rnd((N, d), 9, W.TID_K)
    v = rnd((N, d), 9, W.TID_V)
    p = np.random.default_rng(9).permutation(N)
    o, lse = orc.attention(q, k, v, False, 0.35)
    o2, lse2 = orc.attention(q, k[p].copy(), v[p].copy(), False, 0.35)
    close(o2, o, 1e-13, "permute K,V")
    close(lse2, lse, 1e-13, "permute K,V LSE")
    o3, lse3 = orc.attention(q[p].copy(), k, v, False, 0.35)
    close(o3, o[p], 1e-15, "permute Q")
    close(lse3, lse[p], 1e-15, "permute Q LSE")


def pin_linear_in_v(orc):
    """O(Q, K, aV + bV') = a O(Q, K, V) + b O(Q, K, V'); integer V, V' keep aV + bV' exact."""
    rng = np.random.default_rng(10)
    N, d = 31, 8
    q = rnd((N, d), 10)
    k = rnd((N, d), 10, W.TID_K)
    V1 = rng.integers(-4, 5, (N, d)).astype(np.float64)
    V2 = rng.integers(-4, 5, (N, d)).astype(np.float64)
    for causal in (False, True):
        o1, _ = orc.attention(q, k, bf16(V1), causal, 0.3)
        o2, _ = orc.attention(q, k, bf16(V2), causal, 0.3)
        o3, _ = orc.attention(q, k, bf16(2 * V1 - 3 * V2), causal, 0.3)
        close(o3, 2 * o1 - 3 * o2, 1e-12, f"linear in V causal={causal}")


def pin_tiled_algorithm(orc):
    """The tiled algorithm (outer loop over K/V blocks, running m and l, O renormalised each step)
    equals the plain definition for any block sizes, ragged tails included; LSE = m + ln l."""
    N, d = 45, 16
    q = rnd((N, d), 11)
    k = rnd((N, d), 11, W.TID_K)
    v = rnd((N, d), 11, W.TID_V)
    scale = 0.25
    for causal in (False, True):
        o, lse = orc.attention(q, k, v, causal, scale)
        for Br, Bc in ((1, 1), (3, 5), (7, 3), (16, 16), (45, 45), (64, 8), (5, 64)):
            O, l, m = orc.flash_alg1(q, k, v, causal, scale, Br, Bc)
            close(O, o, 1e-12, f"tiled O Br={Br} Bc={Bc} causal={causal}")
            close(m + np.log(l), lse, 1e-12, f"tiled LSE Br={Br} Bc={Bc} causal={causal}")


def pin_paged_decode(orc):
    """Paged decode = plain attention over the sequence's rows gathered in logical order = the last
    row of causal attention over those rows; shuffling the pool with the table changes nothing."""
    case = W.DecodeCase("pin", S=3, H=2, d=16, lens=[1, 17, 40])
    inp = W.make_decode(case)
    q = W.bf16_bits(inp["q"])
    kp = W.bf16_bits(inp["k_pool"])
    vp = W.bf16_bits(inp["v_pool"])
    table = inp["block_table"].numpy()
    lens = inp["seq_lens"].numpy()
    o, lse = orc.decode_paged(q, kp, vp, table, lens, case.scale)
    for s, L in enumerate(case.lens):
        for h in range(case.H):
            rows = [(int(table[s, t // 16]), t % 16) for t in range(L)]
            Kc = np.stack([kp[b, h, r] for b, r in rows])
            Vc = np.stack([vp[b, h, r] for b, r in rows])
            Qc = np.concatenate([np.zeros((L - 1, case.d), np.uint16), q[s, h][None]], axis=0)
            oc, lc = orc.attention(Qc, Kc, Vc, True, case.scale)
            close(o[s, h], oc[-1], 1e-13, f"paged vs causal last row s={s} h={h}")
            close(lse[s, h], lc[-1], 1e-13, f"paged vs causal last row LSE s={s} h={h}")
            S = case.scale * widen(Kc) @ widen(q[s, h])
            close(o[s, h], sps.softmax(S) @ widen(Vc), 1e-13, f"paged vs scipy s={s} h={h}")
    # relocate: move every physical block b to position pi(b), rewrite the table
    P = kp.shape[0]
    pi = np.random.default_rng(12).permutation(P)
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[pi] = kp
    vp2[pi] = vp
    t2 = np.where(table >= 0, pi[np.maximum(table, 0)], -1).astype(np.int32)
    o2, lse2 = orc.decode_paged(q, kp2, vp2, t2, lens, case.scale)
    close(o2, o, 0.0, "relocated pool O")
    close(lse2, lse, 0.0, "relocated pool LSE")


def _gather(kp, vp, table, s, h, L, page=16):
    rows = [(int(table[s, t // page]), t % page) for t in range(L)]
    return np.stack([kp[b, h, r] for b, r in rows]), np.stack([vp[b, h, r] for b, r in rows])


def pin_paged_prefill(orc):
    """Chunked prefill over a paged cache: query t of the chunk sits at position L - Lq + t; causal
    rows see keys 0 .. L - Lq + t of the gathered context (softmax/logsumexp from scipy); the
    last row is the decode step; Lq = L with the whole context is causal attention over it."""
    case = W.DecodeCase("pinpf", S=3, H=2, d=16, lens=[20, 33, 47])
    for Lq in (1, 7, 20):
        inp = W.make_paged_prefill(case, Lq)
        q = W.bf16_bits(inp["q"])
        kp, vp = W.bf16_bits(inp["k_pool"]), W.bf16_bits(inp["v_pool"])
        table, lens = inp["block_table"].numpy(), inp["seq_lens"].numpy()
        for causal in (True, False):
            o, lse = orc.prefill_paged(q, kp, vp, table, lens, causal, case.scale)
            for s, L in enumerate(case.lens):
                for h in range(case.H):
                    Kc, Vc = _gather(kp, vp, table, s, h, L)
                    S_ = case.scale * widen(q[s, h]) @ widen(Kc).T
                    if causal:
                        for t in range(Lq):
                            S_[t, L - Lq + t + 1:] = -np.inf
                    close(o[s, h], sps.softmax(S_, axis=1) @ widen(Vc), 1e-13,
                          f"paged prefill O Lq={Lq} causal={causal} s={s} h={h}")
                    close(lse[s, h], sps.logsumexp(S_, axis=1), 1e-13,
                          f"paged prefill LSE Lq={Lq} causal={causal} s={s} h={h}")
            if Lq == 1 and causal:
                od, ld = orc.decode_paged(q[:, :, 0].copy(), kp, vp, table, lens, case.scale)
                close(o[:, :, 0], od, 1e-15, "paged prefill Lq=1 vs decode")
                close(lse[:, :, 0], ld, 1e-15, "paged prefill Lq=1 vs decode LSE")
    # Lq = L over one sequence: plain causal attention over the gathered rows
    case1 = W.DecodeCase("pinpf1", S=1, H=2, d=16, lens=[37])
    inp = W.make_paged_prefill(case1, 37)
    q = W.bf16_bits(inp["q"])
    kp, vp = W.bf16_bits(inp["k_pool"]), W.bf16_bits(inp["v_pool"])
    table, lens = inp["block_table"].numpy(), inp["seq_lens"].numpy()
    o, lse = orc.prefill_paged(q, kp, vp, table, lens, True, case1.scale)
    for h in range(2):
        Kc, Vc = _gather(kp, vp, table, 0, h, 37)
        oc, lc = orc.attention(q[0, h].copy(), Kc, Vc, True, case1.scale)
        close(o[0, h], oc, 1e-13, "paged prefill Lq=L vs causal attention")
        close(lse[0, h], lc, 1e-13, "paged prefill Lq=L vs causal attention LSE")


def _fwd_loss(Q, K, V, dO, scale, causal):
    """sum(dO * O) for O = softmax(scale Q K^T, causal) V, fp64 numpy (scipy softmax)."""
    S_ = scale * Q @ K.T
    if causal:
        S_ = np.where(np.tril(np.ones_like(S_, dtype=bool)), S_, -np.inf)
    return float(np.sum(dO * (sps.softmax(S_, axis=1) @ V)))


def pin_bwd_finite_differences(orc):
    """Every entry of dQ, dK, dV equals the central difference of sum(dO * O) (fp64 forward from
    scipy's softmax, step 1e-6; truncation ~1e-12, rounding ~1e-10)."""
    N, d, scale = 6, 4, 0.7
    q, k, v, do = (rnd((N, d), 90 + t) for t in range(4))
    Q, K, V, dO = (widen(x) for x in (q, k, v, do))
    h = 1e-6
    for causal in (False, True):
        dq, dk, dv = orc.attention_bwd(q, k, v, do, causal, scale)
        for name, X, G in (("dQ", Q, dq), ("dK", K, dk), ("dV", V, dv)):
            fd = np.zeros_like(X)
            for idx in np.ndindex(*X.shape):
                Xp, Xm = X.copy(), X.copy()
                Xp[idx] += h
                Xm[idx] -= h
                args_p = [Xp if Y is X else Y for Y in (Q, K, V)]
                args_m = [Xm if Y is X else Y for Y in (Q, K, V)]
                fd[idx] = (_fwd_loss(*args_p, dO, scale, causal) -
                           _fwd_loss(*args_m, dO, scale, causal)) / (2 * h)
            close(G, fd, 1e-7, f"backward {name} vs finite differences causal={causal}")


def pin_bwd_autograd(orc):
    """dQ, dK, dV equal torch.autograd through torch.softmax in fp64, on two heads of N = 70 (a
    subset of heads selects the same values)."""
    B, H, N, d = 1, 2, 70, 16
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (rnd((B, H, N, d), 95 + t) for t in range(4))
    for causal in (False, True):
        Q, K, V = (torch.tensor(widen(x), requires_grad=True) for x in (q, k, v))
        S_ = scale * Q @ K.transpose(-1, -2)
        if causal:
            S_ = S_.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
        O = torch.softmax(S_, dim=-1) @ V
        O.backward(torch.tensor(widen(do)))
        dq, dk, dv = orc.attention_bwd(q, k, v, do, causal, scale)
        for name, g, t in (("dQ", dq, Q), ("dK", dk, K), ("dV", dv, V)):
            close(g, t.grad.numpy(), 1e-12, f"backward {name} vs autograd causal={causal}")
        sq, sk, sv = orc.attention_bwd(q, k, v, do, causal, scale, heads=[1])
        close(sq[0], dq[0, 1], 0.0, "backward head subset dQ")
        close(sv[0], dv[0, 1], 0.0, "backward head subset dV")


def pin_bwd_closed_forms(orc):
    """Rows of P sum to one, so sum_j dV_j = sum_i dO_i and each row of dS sums to zero, giving
    sum_j dK_j = 0.  One key: P = 1, so dQ = dK = 0 and dV = dO.  Q = 0: uniform weights, so every
    dV_j = mean_i dO_i (non-causal).  Adding one vector u to every key leaves all three gradients
    unchanged (the softmax ignores a per-row constant)."""
    N, d, scale = 50, 8, 0.35
    q, k, v, do = (rnd((N, d), 100 + t) for t in range(4))
    for causal in (False, True):
        dq, dk, dv = orc.attention_bwd(q, k, v, do, causal, scale)
        close(dv.sum(axis=0), widen(do).sum(axis=0), 1e-11, f"sum dV = sum dO causal={causal}")
        close(dk.sum(axis=0), np.zeros(d), 1e-11, f"sum dK = 0 causal={causal}")
    q1, k1, v1, do1 = (x[:1].copy() for x in (q, k, v, do))
    dq, dk, dv = orc.attention_bwd(q1, k1, v1, do1, False, scale)
    close(dq, np.zeros((1, d)), 0.0, "one key: dQ = 0")
    close(dk, np.zeros((1, d)), 0.0, "one key: dK = 0")
    close(dv, widen(do1), 0.0, "one key: dV = dO")
    dq, dk, dv = orc.attention_bwd(bf16(np.zeros((N, d))), k, v, do, False, scale)
    close(dv, np.tile(widen(do).mean(axis=0), (N, 1)), 1e-13, "Q = 0: dV_j = mean dO")
    # keys on a coarse grid so that K + u is exact in bf16
    kg = bf16(np.round(widen(k) * 4) / 4)
    ks = bf16(widen(kg) + 0.5 * np.arange(1, d + 1) / d)
    for causal in (False, True):
        a = orc.attention_bwd(q, kg, v, do, causal, scale)
        b = orc.attention_bwd(q, ks, v, do, causal, scale)
        for name, x, y in zip(("dQ", "dK", "dV"), a, b):
            close(x, y, 1e-11, f"key shift leaves {name} unchanged causal={causal}")


def _ancestors_or_self(parents, t):
    seen = set()
    while t >= 0:
        seen.add(t)
        t = parents[t]
    return seen


def pin_tree_attention(orc):
    """Tree verification: node t of a draft tree continues the context along the path root..t, so
    it sees the L - T context tokens and exactly its ancestors and itself among the tree's nodes
    (walked here from the parent lists, not from the masks).  scipy softmax/logsumexp over the
    gathered rows; a chain tree is the causal chunk of the same T tokens; with no context a star
    tree gives each node its own value row; a node that sees nothing gets O = 0, LSE = -inf."""
    case = W.DecodeCase("pintree", S=3, H=2, d=16, lens=[20, 41, 64])
    for shape in ("random", "star", "chain"):
        inp = W.make_tree_verify(case, 12, shape)
        q = W.bf16_bits(inp["q"])
        kp, vp = W.bf16_bits(inp["k_pool"]), W.bf16_bits(inp["v_pool"])
        table, lens = inp["block_table"].numpy(), inp["seq_lens"].numpy()
        o, lse = orc.tree_attention(q, kp, vp, table, lens, inp["tree_mask"].numpy(), case.scale)
        for s, L in enumerate(case.lens):
            ctx = L - 12
            for h in range(case.H):
                Kc, Vc = _gather(kp, vp, table, s, h, L)
                S_ = case.scale * widen(q[s, h]) @ widen(Kc).T
                for t in range(12):
                    vis = _ancestors_or_self(inp["parents"][s], t)
                    for u in range(12):
                        if u not in vis:
                            S_[t, ctx + u] = -np.inf
                close(o[s, h], sps.softmax(S_, axis=1) @ widen(Vc), 1e-13,
                      f"tree {shape} O s={s} h={h}")
                close(lse[s, h], sps.logsumexp(S_, axis=1), 1e-13, f"tree {shape} LSE s={s} h={h}")
        if shape == "chain":
            oc, lc = orc.prefill_paged(q, kp, vp, table, lens, True, case.scale)
            close(o, oc, 0.0, "chain tree vs causal chunk")
            close(lse, lc, 0.0, "chain tree vs causal chunk LSE")
    # no context: a star tree leaves each node only itself
    case0 = W.DecodeCase("pintree0", S=1, H=2, d=16, lens=[9])
    inp = W.make_tree_verify(case0, 9, "star")
    q = W.bf16_bits(inp["q"])
    kp, vp = W.bf16_bits(inp["k_pool"]), W.bf16_bits(inp["v_pool"])
    table, lens = inp["block_table"].numpy(), inp["seq_lens"].numpy()
    o, lse = orc.tree_attention(q, kp, vp, table, lens, inp["tree_mask"].numpy(), case0.scale)
    for h in range(2):
        Kc, Vc = _gather(kp, vp, table, 0, h, 9)
        close(o[0, h], widen(Vc), 0.0, "star without context: O = own V")
        close(lse[0, h], case0.scale * np.sum(widen(q[0, h]) * widen(Kc), axis=1), 1e-13,
              "star without context: LSE = own score")
    # a node that sees nothing
    mask = inp["tree_mask"].numpy().copy()
    mask[0, 4] = 0
    o, lse = orc.tree_attention(q, kp, vp, table, lens, mask, case0.scale)
    close(o[0, :, 4], np.zeros((2, 16)), 0.0, "empty row: O = 0")
    assert np.all(np.isneginf(lse[0, :, 4])), "empty row: LSE = -inf"


def pin_key_ranges_merge(orc):
    """Splitting the keys into ranges and merging the range partials gives plain attention, for
    any split (sequence-length parallelism; the merge is the rescaling rule of the tiled
    algorithm); a range partial is scipy's softmax over that range's visible keys; an empty
    partial (O = 0, LSE = -inf) changes nothing; the merge of log-sum-exps near 1000 stays finite
    and equals scipy's logsumexp."""
    BH, N, d, scale = 2, 70, 16, 0.3
    q, k, v = (rnd((BH, N, d), 120 + t) for t in range(3))
    for causal in (False, True):
        full_o, full_l = orc.attention(q, k, v, causal, scale)
        for cuts in ([35], [1, 69], [10, 30, 31, 60], [70]):
            bounds = [0] + cuts + ([N] if cuts[-1] != N else [])
            parts_o, parts_l = [], []
            for a, b in zip(bounds[:-1], bounds[1:]):
                po, pl = orc.attention_keyrange(q, k[:, a:b].copy(), v[:, a:b].copy(), 0, a, causal,
                                                scale)
                parts_o.append(po)
                parts_l.append(pl)
            mo, ml = orc.merge_partials(np.stack(parts_o), np.stack(parts_l))
            close(mo, full_o, 1e-13, f"merged key ranges {cuts} causal={causal}")
            close(ml, full_l, 1e-13, f"merged key ranges LSE {cuts} causal={causal}")
        # one middle range against scipy, queries at positions 40.. over keys at 20..50
        po, pl = orc.attention_keyrange(q[:, 40:].copy(), k[:, 20:50].copy(), v[:, 20:50].copy(), 40,
                                        20, causal, scale)
        for h in range(BH):
            S_ = scale * widen(q[h, 40:]) @ widen(k[h, 20:50]).T
            if causal:
                for i in range(N - 40):
                    S_[i, (40 + i) - 20 + 1:] = -np.inf
            close(po[h], sps.softmax(S_, axis=1) @ widen(v[h, 20:50]), 1e-13, "range partial O")
            close(pl[h], sps.logsumexp(S_, axis=1), 1e-13, "range partial LSE")
    # causal: queries before the range see nothing
    po, pl = orc.attention_keyrange(q, k[:, 50:].copy(), v[:, 50:].copy(), 0, 50, True, scale)
    close(po[:, :50], np.zeros((BH, 50, d)), 0.0, "no visible key: O = 0")
    assert np.all(np.isneginf(pl[:, :50])), "no visible key: LSE = -inf"
    # neutrality of an empty partial
    o1, l1 = orc.attention(q, k, v, False, scale)
    mo, ml = orc.merge_partials(np.stack([o1, np.zeros_like(o1)]),
                                np.stack([l1, np.full_like(l1, -np.inf)]))
    close(mo, o1, 0.0, "empty partial is neutral")
    close(ml, l1, 0.0, "empty partial is neutral LSE")
    # large log-sum-exps: exact reference from scipy's logsumexp on the weights
    rng = np.random.default_rng(7)
    lp = 1000.0 + rng.normal(size=(3, 5))
    op = rng.normal(size=(3, 5, 4))
    mo, ml = orc.merge_partials(op, lp)
    w = np.exp(lp - sps.logsumexp(lp, axis=0))
    close(mo, np.einsum("gr,grc->rc", w, op), 1e-12, "merge weights at LSE ~ 1000")
    close(ml, sps.logsumexp(lp, axis=0), 1e-12, "merged LSE at ~ 1000")


ALL_PINS = [pin_uniform_scores, pin_single_key, pin_dominant_score, pin_two_keys_logistic,
            pin_shift_invariance, pin_rows_sum_to_one, pin_library_softmax, pin_permutation,
            pin_linear_in_v, pin_tiled_algorithm, pin_paged_decode, pin_paged_prefill,
            pin_bwd_finite_differences, pin_bwd_autograd, pin_bwd_closed_forms,
            pin_tree_attention, pin_key_ranges_merge]
