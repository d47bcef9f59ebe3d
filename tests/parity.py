"""Helpers for the GPU-vs-oracle parity tests: inputs from the shared generator, outputs compared
element by element with the tolerance the acceptance bar states
(max|dO| <= 1e-2, mean|dO| <= 1e-3, max|dLSE| <= 1e-3)."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import workloads as W
from oracle import oracle as orc

TOL_MAX_O = 1e-2
TOL_MEAN_O = 1e-3
TOL_LSE = 1e-3


# bf16 output adds the output format's own rounding: round-to-nearest-even to 8 significant bits
# moves a value by at most 2^-8 of its magnitude (2^-9 on average), on top of the stated bound.
BF16_REL = 2.0 ** -8
# below this magnitude bf16 O must meet the plain max|dO| bound with no rounding allowance
BF16_PLAIN_BELOW = 2.0


def assert_close(o_gpu, lse_gpu, o_ref, lse_ref, what="", out_bf16=False):
    o_gpu = np.asarray(o_gpu, np.float64)
    d = np.abs(o_gpu - o_ref)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    mx, mean = float(d.max()), float(d.mean())
    log = os.environ.get("FA_PARITY_LOG")
    if log:
        dl = (float(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref).max())
              if lse_gpu is not None else None)
        with open(log, "a") as f:
            f.write(json.dumps({"case": what, "out": "bf16" if out_bf16 else "f32",
                                "max_dO": mx, "mean_dO": mean, "max_dLSE": dl,
                                "n": int(d.size)}) + "\n")
    if out_bf16:
        excess = float((d - BF16_REL * np.abs(o_ref)).max())
        assert excess <= TOL_MAX_O, f"{what}: max(|dO| - 2^-8|O|) {excess:.3e} > {TOL_MAX_O}"
        # where |O| < 2 the output's own rounding is below 2^-7 < 1e-2, so the plain bound holds
        # there without the allowance: a regression in the arithmetic cannot hide behind it
        small = np.abs(o_ref) < BF16_PLAIN_BELOW
        if small.any():
            mx_small = float(d[small].max())
            assert mx_small <= TOL_MAX_O, (
                f"{what}: max|dO| {mx_small:.3e} > {TOL_MAX_O} where |O| < {BF16_PLAIN_BELOW}")
        mean_allow = TOL_MEAN_O + float((BF16_REL / 2 * np.abs(o_ref)).mean())
        assert mean <= mean_allow, f"{what}: mean|dO| {mean:.3e} > {mean_allow:.3e}"
    else:
        assert mx <= TOL_MAX_O, f"{what}: max|dO| {mx:.3e} > {TOL_MAX_O}"
        assert mean <= TOL_MEAN_O, f"{what}: mean|dO| {mean:.3e} > {TOL_MEAN_O}"
    if lse_gpu is not None:
        dl = float(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref).max())
        assert dl <= TOL_LSE, f"{what}: max|dLSE| {dl:.3e} > {TOL_LSE}"
    return mx, mean


def sample_rows(case: W.PrefillCase, n_heads: int = 6, n_random: int = 24, seed: int = 1):
    """(bh, row) pairs: a spread of heads; per head rows 0, 127, 128, N-1, every 128-row tile
    boundary (up to 16 of them) and seeded random rows."""
    rng = np.random.default_rng(seed)
    BH, N = case.B * case.H, case.N
    heads = sorted(set([0, BH - 1] + list(rng.integers(0, BH, n_heads))))
    pairs = []
    for bh in heads:
        rows = {0, min(127, N - 1), min(128, N - 1), N - 1}
        bounds = list(range(0, N, 128))
        step = max(1, len(bounds) // 16)
        for b in bounds[::step]:
            rows.update({b, max(0, b - 1)})
        rows.update(int(r) for r in rng.integers(0, N, n_random))
        pairs += [(bh, r) for r in sorted(rows)]
    return np.array(pairs, dtype=np.int64)


def run_prefill(case: W.PrefillCase, out_dtype=torch.float32, full: bool | None = None):
    """Run fa_fwd on the case and compare with the oracle (all rows if small, else sampled)."""
    import exact_attention_158_b200 as fa
    q, k, v = W.make_prefill(case, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=case.causal, scale=case.scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    qb, kb, vb = (W.bf16_bits(t) for t in (q, k, v))
    BH, N, d = case.B * case.H, case.N, case.d
    if full is None:
        full = BH * N * N * d <= 3e9
    if full:
        o_ref, lse_ref = orc.attention(qb.reshape(BH, N, d), kb.reshape(BH, N, d),
                                       vb.reshape(BH, N, d), case.causal, case.scale)
        return assert_close(o.float().cpu().numpy().reshape(BH, N, d), lse.cpu().numpy().reshape(BH, N),
                            o_ref, lse_ref, case.name, out_bf16=out_dtype == torch.bfloat16)
    pairs = sample_rows(case)
    o_ref, lse_ref = orc.attention_rows(qb.reshape(BH, N, d), kb.reshape(BH, N, d),
                                        vb.reshape(BH, N, d), case.causal, case.scale, pairs)
    og = o.float().reshape(BH, N, d)[pairs[:, 0], pairs[:, 1]].cpu().numpy()
    lg = lse.reshape(BH, N)[pairs[:, 0], pairs[:, 1]].cpu().numpy()
    return assert_close(og, lg, o_ref, lse_ref, case.name + " (sampled rows)",
                        out_bf16=out_dtype == torch.bfloat16)


# Backward tolerance.  Each gradient is an fp32 sum of products whose device-formed factor passed
# through bf16 (unit roundoff u = 2^-9): P for dV, and P then dS = P (dP - D) for dK and dQ, with D
# itself formed from the bf16 forward output.  Two roundings of 2^-9 and a cancellation factor of
# up to 4 in the sums give 2^-6 of the tensor's largest magnitude for the worst element, and 2^-7 of
# its mean magnitude on average; 2^-16 absolute covers tensors that are exactly zero (one key).
TOL_GRAD_MAX = 2.0 ** -6
TOL_GRAD_MEAN = 2.0 ** -7
TOL_GRAD_ABS = 2.0 ** -16


def assert_grads_close(got, ref, what="", out_bf16=False):
    """got, ref: dicts name -> array (same shapes).  Per tensor: max|d| <= 2^-6 max|ref| + 2^-16 and
    mean|d| <= 2^-7 mean|ref| + 2^-16; bf16 gradients add their own rounding (2^-8 |ref| per
    element, 2^-9 on average)."""
    out = {}
    for name in ref:
        g = np.asarray(got[name], np.float64)
        r = np.asarray(ref[name], np.float64)
        assert g.shape == r.shape, f"{what} {name}: shape {g.shape} vs {r.shape}"
        assert np.all(np.isfinite(g)), f"{what} {name}: non-finite gradient"
        d = np.abs(g - r)
        if out_bf16:
            d = np.maximum(d - BF16_REL * np.abs(r), 0.0)
        mx, mean = float(d.max()), float(d.mean())
        lim_max = TOL_GRAD_MAX * float(np.abs(r).max()) + TOL_GRAD_ABS
        lim_mean = TOL_GRAD_MEAN * float(np.abs(r).mean()) + TOL_GRAD_ABS
        log = os.environ.get("FA_PARITY_LOG")
        if log:
            with open(log, "a") as f:
                f.write(json.dumps({"case": f"{what} {name}", "out": "bf16" if out_bf16 else "f32",
                                    "max_err": mx, "lim_max": lim_max, "mean_err": mean,
                                    "lim_mean": lim_mean, "n": int(d.size)}) + "\n")
        assert mx <= lim_max, f"{what} {name}: max err {mx:.3e} > {lim_max:.3e}"
        assert mean <= lim_mean, f"{what} {name}: mean err {mean:.3e} > {lim_mean:.3e}"
        out[name] = (mx, mean)
    return out


def run_backward(case: W.PrefillCase, grad_dtype=torch.float32, heads=None, scale=None,
                 o_dtype=torch.bfloat16):
    """fa_fwd (O in o_dtype) then fa_bwd on the case (dO from the shared generator); the listed
    heads (default all) compared with the oracle's backward.  scale: override of 1/sqrt(d)."""
    scale = case.scale if scale is None else scale
    import exact_attention_158_b200 as fa
    q, k, v = W.make_prefill(case, device="cuda")
    do = W.make_dout(case, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, causal=case.causal, scale=scale, out_dtype=o_dtype)
    dq, dk, dv = fa.fa_bwd(q, k, v, o, do, lse, causal=case.causal, scale=scale,
                           grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    BH, N, d = case.B * case.H, case.N, case.d
    if heads is None:
        heads = list(range(BH))
    rq, rk, rv = orc.attention_bwd(*(W.bf16_bits(t).reshape(BH, N, d) for t in (q, k, v, do)),
                                   case.causal, scale, heads=heads)
    pick = lambda t: t.float().reshape(BH, N, d)[heads].cpu().numpy()
    return assert_grads_close({"dq": pick(dq), "dk": pick(dk), "dv": pick(dv)},
                              {"dq": rq, "dk": rk, "dv": rv},
                              f"{case.name} o={'f32' if o_dtype == torch.float32 else 'bf16'}",
                              out_bf16=grad_dtype == torch.bfloat16)
