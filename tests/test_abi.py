"""The C-ABI library: it loads, exports every symbol include/fa.h declares, and its host-side
argument checks reject bad calls before anything is launched (no GPU needed)."""
import ctypes
import os
import re

import pytest

import exact_attention_158_b200 as fa
from exact_attention_158_b200 import build as fab

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    fab.build()
    return fa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_functions() == sorted(fa.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from {fa.library_path()}"


def test_status_strings_and_version(lib):
    for code, name in fa.STATUS.items():
        assert lib.fa_status_string(code).decode().startswith(name)
    assert lib.fa_version() >= 100


# fake device addresses: never dereferenced, every call below fails its host-side checks first
A = 1 << 20


def fwd(lib, q=A, k=2 * A, v=3 * A, o=4 * A, dt=0, lse=None, B=1, H=1, N=8, d=64, causal=0,
        scale=0.0):
    return lib.fa_fwd(q, k, v, o, dt, lse, B, H, N, d, causal, scale, None)


def test_fwd_rejects_bad_arguments(lib):
    assert fwd(lib, q=None) == 1
    assert fwd(lib, B=0) == 1 and fwd(lib, H=0) == 1 and fwd(lib, N=0) == 1
    assert fwd(lib, causal=2) == 1
    assert fwd(lib, dt=7) == 1
    assert fwd(lib, d=96) == 2 and fwd(lib, d=256) == 2
    assert fwd(lib, scale=float("nan")) == 1 and fwd(lib, scale=float("inf")) == 1
    assert fwd(lib, q=A + 8) == 3 and fwd(lib, o=4 * A + 4) == 3
    assert fwd(lib, lse=5 * A + 2) == 3
    # output overlapping an input
    assert fwd(lib, o=A + 16) == 1
    assert fwd(lib, lse=2 * A + 64) == 1
    # more work units (pairs of 128-row query tiles) than an int counts: B*H = 2^30, 64 pairs each
    # (buffers far apart, so only the unit count is wrong)
    far = 1 << 52
    assert lib.fa_fwd(far, 2 * far, 3 * far, 4 * far, 0, None, 1 << 15, 1 << 15, 1 << 14, 64, 0,
                      0.0, None) == 1


def dec(lib, ws=8 * A, ws_bytes=1 << 30, S=2, H=2, d=128, maxb=4, P=8, table=5 * A, lens=6 * A,
        q=A, o=7 * A, lse=None):
    return lib.fa_decode_paged(q, 2 * A, 3 * A, table, maxb, lens, P, o, 0, lse, S, H, d, 0.0, ws,
                               ws_bytes, None)


def test_decode_workspace_and_rejections(lib):
    need = lib.fa_decode_workspace_size(64, 32, 128, 512)
    assert need == 64 * 32 * 16 * (128 + 2) * 4  # 512 blocks -> 16 chunks of 32 blocks
    assert lib.fa_decode_workspace_size(0, 32, 128, 512) == 0
    assert lib.fa_decode_workspace_size(1, 1, 96, 1) == 0
    assert dec(lib, ws=None) == 6
    assert dec(lib, ws_bytes=16) == 6
    assert dec(lib, S=0) == 1 and dec(lib, maxb=0) == 1 and dec(lib, P=0) == 1
    assert dec(lib, d=80) == 2
    assert dec(lib, table=5 * A + 2) == 3
    assert dec(lib, ws=8 * A + 8) == 3
    assert dec(lib, o=8 * A) == 1  # output overlaps the workspace


def pp(lib, q=A, table=5 * A, maxb=4, lens=6 * A, P=8, o=7 * A, dt=0, lse=None, S=2, H=2, Lq=16,
       d=128, causal=1, scale=0.0):
    return lib.fa_prefill_paged(q, 2 * A, 3 * A, table, maxb, lens, P, o, dt, lse, S, H, Lq, d,
                                causal, scale, None)


def test_prefill_paged_rejections(lib):
    assert pp(lib, q=None) == 1 and pp(lib, table=None) == 1 and pp(lib, lens=None) == 1
    assert pp(lib, S=0) == 1 and pp(lib, Lq=0) == 1 and pp(lib, maxb=0) == 1 and pp(lib, P=0) == 1
    assert pp(lib, Lq=4 * 16 + 1) == 1  # the chunk cannot be longer than a table row maps
    assert pp(lib, causal=3) == 1 and pp(lib, dt=9) == 1
    assert pp(lib, d=96) == 2
    assert pp(lib, scale=float("nan")) == 1
    assert pp(lib, q=A + 8) == 3 and pp(lib, table=5 * A + 2) == 3 and pp(lib, lens=6 * A + 1) == 3
    assert pp(lib, o=A + 32) == 1  # output overlaps q
    assert pp(lib, o=2 * A + 64) == 1  # output overlaps the K pool
    # (block, head) pages are indexed as block * H + head in an int: (num_blocks + 1) * H must fit
    assert pp(lib, P=2 ** 30, H=2) == 1


def bwd(lib, dq=8 * A, ws=12 * A, ws_bytes=1 << 30, B=1, H=2, N=300, d=128, causal=0, dt=0,
        lse=6 * A, scale=0.0, odt=0):
    return lib.fa_bwd(A, 2 * A, 3 * A, 4 * A, odt, 5 * A, lse, dq, 9 * A, 10 * A, dt, B, H, N, d,
                      causal, scale, ws, ws_bytes, None)


def test_bwd_workspace_and_rejections(lib):
    # N = 300 pads to 384 rows: dQ accumulator (d floats) + LSE2 + D per row
    assert lib.fa_bwd_workspace_size(1, 2, 300, 128) == 2 * 384 * (128 + 2) * 4
    assert lib.fa_bwd_workspace_size(1, 2, 300, 80) == 0
    assert lib.fa_bwd_workspace_size(0, 2, 300, 64) == 0
    assert bwd(lib, ws=None) == 6 and bwd(lib, ws_bytes=1000) == 6
    assert bwd(lib, B=0) == 1 and bwd(lib, N=0) == 1 and bwd(lib, causal=5) == 1
    assert bwd(lib, dt=3) == 1 and bwd(lib, lse=None) == 1 and bwd(lib, odt=2) == 1
    assert bwd(lib, d=32) == 2
    assert bwd(lib, dq=8 * A + 8) == 3 and bwd(lib, lse=6 * A + 2) == 3 and bwd(lib, ws=12 * A + 4) == 3
    assert bwd(lib, dq=A + 1024) == 1   # dQ overlaps q
    assert bwd(lib, dq=9 * A + 64) == 1  # dQ overlaps dK
    assert bwd(lib, ws=10 * A + 64) == 1  # workspace overlaps dV


def test_tree_attention_rejections(lib):
    def tree(mask=11 * A, T=8, S=2, o=7 * A, d=128):
        return lib.fa_tree_attention(A, 2 * A, 3 * A, 5 * A, 4, 6 * A, 8, mask, o, 0, None, S, 2,
                                     T, d, 0.0, None)
    assert tree(mask=None) == 1
    assert tree(T=0) == 1 and tree(T=65) == 1
    assert tree(mask=11 * A + 4) == 3
    assert tree(o=11 * A - 64) == 1  # output overlaps the mask
    assert tree(d=96) == 2


def test_keyrange_and_merge_rejections(lib):
    def kr(q_row0=0, Nk=64, k_pos0=0, Nq=100, d=128, o=7 * A, causal=0):
        return lib.fa_fwd_keyrange(A, 2 * A, 3 * A, o, 1, 8 * A, 1, 2, Nq, q_row0, Nk, k_pos0, d,
                                   causal, 0.0, None)
    assert kr(q_row0=100) == 1 and kr(q_row0=-1) == 1 and kr(Nk=0) == 1 and kr(k_pos0=-5) == 1
    assert kr(causal=2) == 1 and kr(d=32) == 2
    far = 1 << 52  # unit count past an int, buffers far apart
    assert lib.fa_fwd_keyrange(far, 2 * far, 3 * far, 4 * far, 1, None, 1 << 15, 1 << 15, 1 << 14, 0,
                               64, 0, 128, 0, 0.0, None) == 1
    assert kr(o=A + 64) == 1  # output overlaps q
    assert lib.fa_fwd_keyrange(A, 2 * A, 3 * A, 7 * A, 1, 2 * A + 64, 1, 2, 100, 0, 64, 0, 128, 0,
                               0.0, None) == 1  # LSE overlaps k
    def mg(G=2, rows=10, d=64, o=5 * A, parts=A):
        return lib.fa_merge_partials(parts, 3 * A, G, rows, d, o, 0, None, None)
    assert mg(G=0) == 1 and mg(rows=0) == 1 and mg(d=96) == 2
    assert mg(parts=A + 4) == 3
    assert mg(o=A + 128) == 1  # output overlaps the partials


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fa_fwd(x, x, x)
