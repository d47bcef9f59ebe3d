"""fa_decode_paged_noalloc, the decode entry point for callers that cannot allocate device memory
(for example an engine whose allocator already owns nearly all of the GPU for its KV-cache pool,
or a decode loop that cannot pay for cudaMalloc's latency and synchronisation).  Its scratch is a
static device array inside the library.  Checked through the C ABI against fa_decode_paged (which
takes a caller workspace) and against the fp64 oracle on two calls in a row, the second one reusing
the array the first call left behind, and for its size limit; the Python wrapper is checked for the
same results and for rejecting wrongly shaped buffers before anything reaches the library.

This file sorts last so that a run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from exact_attention_158_b200 import build as fab
    import exact_attention_158_b200 as fa
    fab.build()
    lib = fa.load_library()
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.fa_decode_paged_noalloc.argtypes = [vp, vp, vp, vp, i32, vp, i32, vp, i32, vp, i32, i32,
                                            i32, ctypes.c_float, vp]
    lib.fa_decode_paged_noalloc.restype = i32
    return lib


def call_noalloc(lib, inp, case, o, lse):
    stream = torch.cuda.current_stream().cuda_stream
    code = 1 if o.dtype == torch.float32 else 0
    return lib.fa_decode_paged_noalloc(
        inp["q"].data_ptr(), inp["k_pool"].data_ptr(), inp["v_pool"].data_ptr(),
        inp["block_table"].data_ptr(), inp["block_table"].shape[1], inp["seq_lens"].data_ptr(),
        inp["num_blocks"], o.data_ptr(), code, lse.data_ptr(), case.S, case.H, case.d, 0.0,
        stream)


def oracle_decode(inp, case):
    return orc.decode_paged(W.bf16_bits(inp["q"]), W.bf16_bits(inp["k_pool"]),
                            W.bf16_bits(inp["v_pool"]), inp["block_table"].cpu().numpy(),
                            inp["seq_lens"].cpu().numpy(), case.scale)


def test_noalloc_matches_workspace_entry_point_twice(lib):
    import exact_attention_158_b200 as fa
    cases = [W.DecodeCase("noalloc_a", S=6, H=8, d=128, lens=[1, 700, 4096, 17, 2500, 8192]),
             W.DecodeCase("noalloc_b", S=9, H=4, d=64, lens=[33, 1, 6000, 512, 513, 15, 16, 3000, 90])]
    for case in cases:  # two calls in a row; the second finds the first call's scratch contents
        inp = W.make_decode(case, device="cuda")
        o_ref, lse_ref = fa.fa_decode_paged(inp["q"], inp["k_pool"], inp["v_pool"],
                                            inp["block_table"], inp["seq_lens"],
                                            out_dtype=torch.float32)
        o = torch.full((case.S, case.H, case.d), float("nan"), device="cuda")
        lse = torch.full((case.S, case.H), float("nan"), device="cuda")
        assert call_noalloc(lib, inp, case, o, lse) == 0
        torch.cuda.synchronize()
        assert fa.device_status() == 0
        parity.assert_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref.cpu().numpy().astype(np.float64),
                            lse_ref.cpu().numpy().astype(np.float64), case.name)
        # and the plain definition itself (fp64 oracle over the gathered pages)
        o_or, lse_or = oracle_decode(inp, case)
        parity.assert_close(o.cpu().numpy(), lse.cpu().numpy(), o_or, lse_or, case.name + " vs oracle")


def test_noalloc_rejects_sizes_beyond_its_array(lib):
    import exact_attention_158_b200 as fa
    A = 1 << 20  # never dereferenced: the size check fails before anything is looked up or launched
    need = lib.fa_decode_workspace_size(64, 32, 128, 2048)
    assert need > fa.NOALLOC_SCRATCH_BYTES
    st = lib.fa_decode_paged_noalloc(A, 2 * A, 3 * A, 4 * A, 2048, 5 * A, 100, 6 * A, 0, None,
                                     64, 32, 128, 0.0, None)
    assert st == 6  # FA_ERR_WORKSPACE
    assert str(need) in lib.fa_last_error_string().decode()
    assert lib.fa_decode_workspace_size(64, 32, 128, 512) <= fa.NOALLOC_SCRATCH_BYTES


def test_noalloc_python_wrapper(lib):
    # the binding's wrapper: same results as the C entry point (bf16 O, then fp32 O without an
    # LSE buffer), on the current stream
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("noalloc_py", S=5, H=8, d=128, lens=[1, 129, 3000, 64, 777])
    inp = W.make_decode(case, device="cuda")
    o_or, lse_or = oracle_decode(inp, case)
    o = torch.empty((case.S, case.H, case.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((case.S, case.H), dtype=torch.float32, device="cuda")
    fa.fa_decode_paged_noalloc(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                               inp["seq_lens"], o, lse)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    parity.assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_or, lse_or,
                        "noalloc wrapper bf16", out_bf16=True)
    o32 = torch.empty((case.S, case.H, case.d), dtype=torch.float32, device="cuda")
    _, none = fa.fa_decode_paged_noalloc(inp["q"], inp["k_pool"], inp["v_pool"],
                                         inp["block_table"], inp["seq_lens"], o32)
    torch.cuda.synchronize()
    assert none is None
    parity.assert_close(o32.cpu().numpy(), None, o_or, None, "noalloc wrapper f32")


def test_noalloc_python_wrapper_rejects_bad_shapes(lib):
    # wrongly shaped buffers would make the kernels read or write past them: the wrapper refuses
    # them before calling the library
    import exact_attention_158_b200 as fa
    case = W.DecodeCase("noalloc_bad", S=3, H=4, d=64, lens=[10, 200, 33])
    inp = W.make_decode(case, device="cuda")
    args = [inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"], inp["seq_lens"]]
    good_o = torch.empty((3, 4, 64), dtype=torch.float32, device="cuda")
    bad = [
        dict(out=torch.empty((3, 4, 32), dtype=torch.float32, device="cuda")),
        dict(out=torch.empty((2, 4, 64), dtype=torch.float32, device="cuda")),
        dict(out=good_o, lse=torch.empty((3, 5), dtype=torch.float32, device="cuda")),
        dict(out=good_o, lse=torch.empty((3, 4), dtype=torch.float64, device="cuda")),
        dict(out=torch.empty((3, 4, 64), dtype=torch.float16, device="cuda")),
    ]
    for kw in bad:
        with pytest.raises(ValueError):
            fa.fa_decode_paged_noalloc(*args, **kw)
    with pytest.raises(ValueError):  # block table with fewer rows than sequences
        fa.fa_decode_paged_noalloc(inp["q"], inp["k_pool"], inp["v_pool"],
                                   inp["block_table"][:2].contiguous(), inp["seq_lens"], good_o)
    with pytest.raises(ValueError):  # pool of the wrong head count
        fa.fa_decode_paged_noalloc(inp["q"], inp["k_pool"][:, :2].contiguous(),
                                   inp["v_pool"][:, :2].contiguous(), inp["block_table"],
                                   inp["seq_lens"], good_o)
