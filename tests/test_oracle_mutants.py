"""Each plausible mistake planted in a copy of the oracle (dropped term, wrong sign or index,
transposed operand, off-by-one mask, wrong page index) must fail at least one pin.  The copies are
compiled on the CPU into a temporary directory; the committed oracle is untouched."""
import os
import subprocess

import pytest

from oracle import oracle as orc
from tests import pins

SRC = os.path.join(os.path.dirname(orc.__file__), "oracle.c")

MUTANTS = {
    "scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
    "exp_sign": ("s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);"),
    "no_max_shift_in_lse": ("*lse = m + log(l);", "*lse = log(l);"),
    "lse_no_log": ("*lse = m + log(l);", "*lse = m + l;"),
    "no_normalise": ("o[c] /= l;", "o[c] /= 1.0;"),
    "score_uses_v": ("widen_bf16(q[k]) * widen_bf16(krow[j][k])",
                     "widen_bf16(q[k]) * widen_bf16(vrow[j][k])"),
    "causal_excludes_diagonal": ("int64_t n_keys = jb->causal ? i + 1 : N;",
                                 "int64_t n_keys = jb->causal ? (i > 0 ? i : 1) : N;"),
    "causal_ignored": ("int64_t n_keys = jb->causal ? i + 1 : N;", "int64_t n_keys = N;"),
    "value_row_index": ("o[c] += s[j] * widen_bf16(vrow[j][c]);",
                        "o[c] += s[j] * widen_bf16(vrow[n_keys - 1 - j][c]);"),
    "page_slot_index": ("int64_t off = ((blk * H + h) * page + t % page) * d;",
                        "int64_t off = ((blk * H + h) * page + t / page % page) * d;"),
    "page_head_index": ("int64_t off = ((blk * H + h) * page + t % page) * d;",
                        "int64_t off = ((h * H + blk % H) * page + t % page) * d;"),
    "tiled_old_weight": ("O[qi * d + e] = (l[qi] * a_old * O[qi * d + e] + a_new * PV[e]) / l_new;",
                         "O[qi * d + e] = (a_old * O[qi * d + e] + a_new * PV[e]) / l_new;"),
    "tiled_l_update": ("double l_new = a_old * l[qi] + a_new * lt;",
                       "double l_new = l[qi] + a_new * lt;"),
    "tiled_mask_edge": ("vis = last + 1;", "vis = last > 0 ? last : 1;"),
    "probs_no_norm": ("row[j] /= l;", "row[j] /= 1.0;"),
    "chunk_causal_offset": ("int64_t n_keys = jb->causal ? L - Lq + t + 1 : L;",
                            "int64_t n_keys = jb->causal ? L - Lq + t : L;"),
    "chunk_query_row": ("attend_row(jb->q + r * d, kr, vr, n_keys, d, jb->scale, s, jb->o + r * d, jb->lse + r);",
                        "attend_row(jb->q + (r - t) * d, kr, vr, n_keys, d, jb->scale, s, jb->o + r * d, jb->lse + r);"),
    "bwd_no_jacobian_mean": ("double ds = p[j] * (dp[j] - pdp);", "double ds = p[j] * dp[j];"),
    "bwd_dv_weight": ("dv[j * d + c] += p[j] * widen_bf16(doi[c]);",
                      "dv[j * d + c] += ds * widen_bf16(doi[c]);"),
    "bwd_dq_scale": ("dq[i * d + c] += scale * ds * widen_bf16(K[j * d + c]);",
                     "dq[i * d + c] += ds * widen_bf16(K[j * d + c]);"),
    "bwd_dk_operand": ("dk[j * d + c] += scale * ds * widen_bf16(qi[c]);",
                       "dk[j * d + c] += scale * ds * widen_bf16(K[j * d + c]);"),
    "bwd_dp_operand": ("acc += widen_bf16(doi[c]) * widen_bf16(V[j * d + c]);",
                       "acc += widen_bf16(doi[c]) * widen_bf16(K[j * d + c]);"),
    "bwd_causal_ignored": ("const int64_t n_keys = causal ? i + 1 : N; /* the keys row i sees */",
                           "const int64_t n_keys = N;"),
    "bwd_row_not_normalised": ("            p[j] /= l;\n        /* dP row", "            p[j] /= 1.0;\n        /* dP row"),
    "tree_mask_ignored": ("if (key >= ctx && !((m >> (key - ctx)) & 1u))", "if (0)"),
    "tree_offset": ("int64_t L = jb->lens[sq], ctx = L - T;", "int64_t L = jb->lens[sq], ctx = L - T + 1;"),
    "tree_bit_order": ("if (key >= ctx && !((m >> (key - ctx)) & 1u))",
                       "if (key >= ctx && !((m >> (T - 1 - (key - ctx))) & 1u))"),
    "range_causal_offset": ("int64_t last = jb->q0 + i - jb->k0;", "int64_t last = jb->q0 + i - jb->k0 - 1;"),
    "merge_weight_sign": ("double w = exp(lse_parts[g * rows + r] - M);", "double w = exp(M - lse_parts[g * rows + r]);"),
    "merge_no_shift": ("double w = exp(lse_parts[g * rows + r] - M);", "double w = exp(lse_parts[g * rows + r]);"),
    "merge_lse_no_log": ("lse[r] = M + log(wsum);", "lse[r] = M + wsum;"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "oracle_mut.c"
    src.write_text(source.replace(old, new))
    lib = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", str(lib), str(src),
                           "-lm", "-lpthread"])
    mutant = orc.OracleLib(str(lib))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, FloatingPointError) as e:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
