"""Exact attention forward for NVIDIA B200 (sm_100a): Python binding of ``libfa_b200.so``.

The functions here only marshal arguments (pointers, sizes, the current CUDA stream) into the C ABI
of include/fa.h; every step of the attention runs in the library's CUDA kernels.  PyTorch supplies
device memory and streams.  There is no fallback: if the library is missing or the device is not
an sm_100 GPU, calls raise.

    o, lse = fa_fwd(q, k, v, causal=True)            # q, k, v: bf16 [B, H, N, d] on cuda
    o, lse = fa_decode_paged(q, k_pool, v_pool, block_table, seq_lens)
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

__all__ = ["fa_fwd", "fa_bwd", "fa_decode_paged", "fa_decode_paged_noalloc", "fa_prefill_paged",
           "fa_tree_attention", "fa_fwd_keyrange", "fa_merge_partials",
           "fa_decode_workspace_size",
           "NOALLOC_SCRATCH_BYTES", "device_status",
           "FaError", "library_path", "load_library", "EXPORTED_SYMBOLS", "STATUS"]

STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_ALIGNMENT",
          4: "FA_ERR_LAUNCH", 5: "FA_ERR_TIMEOUT", 6: "FA_ERR_WORKSPACE"}
FA_OUT_BF16, FA_OUT_F32 = 0, 1

EXPORTED_SYMBOLS = ("fa_fwd", "fa_decode_workspace_size", "fa_decode_paged",
                    "fa_decode_paged_noalloc", "fa_prefill_paged", "fa_tree_attention",
                    "fa_fwd_keyrange", "fa_merge_partials",
                    "fa_bwd_workspace_size",
                    "fa_bwd", "fa_get_device_status",
                    "fa_status_string",
                    "fa_last_error_string", "fa_version", "fa_selftest_wait_timeout",
                    "fa_probe_ex2_rate", "fa_probe_read_rate", "fa_fwd_schedule")

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if _lib is not None:
            msg = f"{where}: {_lib.fa_status_string(status).decode()}"
            if status == 4:
                msg += f" ({_lib.fa_last_error_string().decode()})"
        super().__init__(msg)


def library_path() -> str:
    return _build.LIB_PATH


def load_library():
    """Load the in-tree shared library (build it first with ``python -m exact_attention_158_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} is missing "
                          "(run `python -m exact_attention_158_b200.build`)")
    lib = ctypes.CDLL(path)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, f32, vp]
    lib.fa_fwd.restype = i32
    lib.fa_decode_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.fa_decode_workspace_size.restype = sz
    lib.fa_decode_paged.argtypes = [vp, vp, vp, vp, i32, vp, i32, vp, i32, vp, i32, i32, i32, f32,
                                    vp, sz, vp]
    lib.fa_decode_paged.restype = i32
    lib.fa_prefill_paged.argtypes = [vp, vp, vp, vp, i32, vp, i32, vp, i32, vp, i32, i32, i32, i32,
                                     i32, f32, vp]
    lib.fa_prefill_paged.restype = i32
    lib.fa_fwd_keyrange.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i32,
                                    i32, f32, vp]
    lib.fa_fwd_keyrange.restype = i32
    lib.fa_merge_partials.argtypes = [vp, vp, i32, ctypes.c_longlong, i32, vp, i32, vp, vp]
    lib.fa_merge_partials.restype = i32
    lib.fa_tree_attention.argtypes = [vp, vp, vp, vp, i32, vp, i32, vp, vp, i32, vp, i32, i32, i32,
                                      i32, f32, vp]
    lib.fa_tree_attention.restype = i32
    lib.fa_bwd_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                           f32, vp, ctypes.c_size_t, vp]
    lib.fa_bwd.restype = i32
    lib.fa_get_device_status.argtypes = [vp]
    lib.fa_get_device_status.restype = i32
    lib.fa_status_string.argtypes = [i32]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_error_string.argtypes = []
    lib.fa_last_error_string.restype = ctypes.c_char_p
    lib.fa_version.argtypes = []
    lib.fa_version.restype = i32
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise FaError(status, where)


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _require(t: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out_code(out_dtype) -> int:
    if out_dtype == torch.bfloat16:
        return FA_OUT_BF16
    if out_dtype == torch.float32:
        return FA_OUT_F32
    raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")


def fa_fwd(q, k, v, causal: bool = False, scale: float | None = None,
           out_dtype=torch.bfloat16, out=None, lse=None, return_lse: bool = True, stream=None):
    """Exact attention forward.  q, k, v: bf16 [B, H, N, d] contiguous on one CUDA device.

    Returns (o [B, H, N, d] in out_dtype, lse fp32 [B, H, N] or None)."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n)
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one shape [B, H, N, d]")
    B, H, N, d = q.shape
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    else:
        _require(out, "out", out_dtype)
        if out.shape != q.shape:
            raise ValueError("out has the wrong shape")
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _require(lse, "lse", torch.float32)
        if lse.shape != (B, H, N):
            raise ValueError("lse has the wrong shape")
    with torch.cuda.device(q.device):
        st = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), code,
                        lse.data_ptr() if lse is not None else None, B, H, N, d, int(causal),
                        float(scale) if scale is not None else 0.0, _stream_handle(stream))
    _check(st, "fa_fwd")
    return out, lse


def fa_decode_workspace_size(num_seqs: int, H: int, d: int, max_blocks_per_seq: int) -> int:
    return int(load_library().fa_decode_workspace_size(num_seqs, H, d, max_blocks_per_seq))


def fa_decode_paged(q, k_pool, v_pool, block_table, seq_lens, scale: float | None = None,
                    out_dtype=torch.bfloat16, out=None, lse=None, return_lse: bool = True,
                    workspace=None, stream=None):
    """One decode step over a paged KV cache.

    q bf16 [S, H, d]; k_pool, v_pool bf16 [num_blocks, H, 16, d]; block_table int32
    [S, max_blocks]; seq_lens int32 [S].  Returns (o [S, H, d], lse fp32 [S, H] or None)."""
    lib = load_library()
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _require(t, n)
    _require(block_table, "block_table", torch.int32)
    _require(seq_lens, "seq_lens", torch.int32)
    S, H, d = q.shape
    P = k_pool.shape[0]
    if k_pool.shape != (P, H, 16, d) or v_pool.shape != k_pool.shape:
        raise ValueError("k_pool / v_pool must be [num_blocks, H, 16, d]")
    if block_table.dim() != 2 or block_table.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_table must be [S, max_blocks] and seq_lens [S]")
    maxb = block_table.shape[1]
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty((S, H, d), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((S, H), dtype=torch.float32, device=q.device)
    need = lib.fa_decode_workspace_size(S, H, d, maxb)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.fa_decode_paged(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                 block_table.data_ptr(), maxb, seq_lens.data_ptr(), P,
                                 out.data_ptr(), code,
                                 lse.data_ptr() if lse is not None else None, S, H, d,
                                 float(scale) if scale is not None else 0.0,
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                 _stream_handle(stream))
    _check(st, "fa_decode_paged")
    return out, lse


def fa_bwd(q, k, v, o, dout, lse, causal: bool = False, scale: float | None = None,
           grad_dtype=torch.bfloat16, workspace=None, stream=None):
    """Attention backward: q, k, v, dout bf16 [B, H, N, d]; o (bf16 or fp32) and lse (fp32
    [B, H, N]) from fa_fwd with the same causal and scale.  Returns (dq, dk, dv) in grad_dtype."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _require(t, n)
    if o.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"o must be bf16 or fp32, got {o.dtype}")
    _require(o, "o", o.dtype)
    _require(lse, "lse", torch.float32)
    B, H, N, d = q.shape
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        if t.shape != q.shape:
            raise ValueError(f"{n} must have the shape of q")
    if lse.shape != (B, H, N):
        raise ValueError("lse must be [B, H, N]")
    code = _out_code(grad_dtype)
    need = int(lib.fa_bwd_workspace_size(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk, dv = (torch.empty(q.shape, dtype=grad_dtype, device=q.device) for _ in range(3))
    with torch.cuda.device(q.device):
        st = lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _out_code(o.dtype),
                        dout.data_ptr(),
                        lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), code, B, H, N,
                        d, int(causal), float(scale) if scale is not None else 0.0,
                        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                        _stream_handle(stream))
    _check(st, "fa_bwd")
    return dq, dk, dv


def fa_fwd_keyrange(q, k, v, q_row0: int = 0, k_pos0: int = 0, causal: bool = False,
                    scale: float | None = None, out_dtype=torch.float32, out=None, lse=None,
                    stream=None):
    """Partial attention of the query rows q_row0.. of q [B, H, Nq, d] (row i at position i) over
    the keys k, v [B, H, Nk, d] at positions k_pos0...  Rows that see no key get O = 0,
    LSE = -inf; rows before q_row0 of out / lse are left as they are.  Returns (o, lse)."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if k.shape != (B, H, Nk, d) or v.shape != k.shape:
        raise ValueError("k, v must be [B, H, Nk, d] with q's B, H, d")
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.fa_fwd_keyrange(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), code,
                                 lse.data_ptr(), B, H, Nq, q_row0, Nk, k_pos0, d, int(causal),
                                 float(scale) if scale is not None else 0.0, _stream_handle(stream))
    _check(st, "fa_fwd_keyrange")
    return out, lse


def fa_merge_partials(o_parts, lse_parts, out_dtype=torch.bfloat16, stream=None):
    """o_parts fp32 [G, ..., d], lse_parts fp32 [G, ...]: partials of the same rows over disjoint
    key ranges.  Returns the merged (o [..., d], lse [...])."""
    lib = load_library()
    _require(o_parts, "o_parts", torch.float32)
    _require(lse_parts, "lse_parts", torch.float32)
    G, d = o_parts.shape[0], o_parts.shape[-1]
    if lse_parts.shape != o_parts.shape[:-1]:
        raise ValueError("lse_parts must be o_parts' shape without the last dimension")
    rows = lse_parts[0].numel()
    code = _out_code(out_dtype)
    o = torch.empty(o_parts.shape[1:], dtype=out_dtype, device=o_parts.device)
    lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    with torch.cuda.device(o_parts.device):
        st = lib.fa_merge_partials(o_parts.data_ptr(), lse_parts.data_ptr(), G, rows, d,
                                   o.data_ptr(), code, lse.data_ptr(), _stream_handle(stream))
    _check(st, "fa_merge_partials")
    return o, lse


def fa_tree_attention(q, k_pool, v_pool, block_table, seq_lens, tree_mask,
                      scale: float | None = None, out_dtype=torch.bfloat16, out=None, lse=None,
                      return_lse: bool = True, stream=None):
    """Tree verification: q bf16 [S, H, T, d] holds the T draft nodes, the last T cached tokens of
    each sequence; tree_mask int64 [S, T] (uint64 bit patterns: bit u of entry t set when node t
    sees node u; T <= 64).  Pools, table and lengths as for fa_prefill_paged.
    Returns (o [S, H, T, d], lse fp32 [S, H, T] or None)."""
    lib = load_library()
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _require(t, n)
    _require(block_table, "block_table", torch.int32)
    _require(seq_lens, "seq_lens", torch.int32)
    _require(tree_mask, "tree_mask", torch.int64)
    S, H, T, d = q.shape
    P = k_pool.shape[0]
    if k_pool.shape != (P, H, 16, d) or v_pool.shape != k_pool.shape:
        raise ValueError("k_pool / v_pool must be [num_blocks, H, 16, d]")
    if block_table.dim() != 2 or block_table.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_table must be [S, max_blocks] and seq_lens [S]")
    if tree_mask.shape != (S, T):
        raise ValueError("tree_mask must be [S, T]")
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty((S, H, T, d), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((S, H, T), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.fa_tree_attention(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                   block_table.data_ptr(), block_table.shape[1], seq_lens.data_ptr(),
                                   P, tree_mask.data_ptr(), out.data_ptr(), code,
                                   lse.data_ptr() if lse is not None else None, S, H, T, d,
                                   float(scale) if scale is not None else 0.0,
                                   _stream_handle(stream))
    _check(st, "fa_tree_attention")
    return out, lse


def fa_prefill_paged(q, k_pool, v_pool, block_table, seq_lens, causal: bool = True,
                     scale: float | None = None, out_dtype=torch.bfloat16, out=None, lse=None,
                     return_lse: bool = True, stream=None):
    """Chunked prefill over a paged KV cache: q bf16 [S, H, Lq, d] holds the last Lq positions of
    each sequence (their keys/values already in the cache); k_pool, v_pool bf16
    [num_blocks, H, 16, d]; block_table int32 [S, max_blocks]; seq_lens int32 [S] (each >= Lq).
    Returns (o [S, H, Lq, d], lse fp32 [S, H, Lq] or None)."""
    lib = load_library()
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _require(t, n)
    _require(block_table, "block_table", torch.int32)
    _require(seq_lens, "seq_lens", torch.int32)
    S, H, Lq, d = q.shape
    P = k_pool.shape[0]
    if k_pool.shape != (P, H, 16, d) or v_pool.shape != k_pool.shape:
        raise ValueError("k_pool / v_pool must be [num_blocks, H, 16, d]")
    if block_table.dim() != 2 or block_table.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_table must be [S, max_blocks] and seq_lens [S]")
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty((S, H, Lq, d), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((S, H, Lq), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.fa_prefill_paged(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
                                  block_table.data_ptr(), block_table.shape[1], seq_lens.data_ptr(),
                                  P, out.data_ptr(), code,
                                  lse.data_ptr() if lse is not None else None, S, H, Lq, d,
                                  int(causal), float(scale) if scale is not None else 0.0,
                                  _stream_handle(stream))
    _check(st, "fa_prefill_paged")
    return out, lse


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the library's device status word."""
    return int(load_library().fa_get_device_status(_stream_handle(stream)))


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def fa_decode_paged_noalloc(q, k_pool, v_pool, block_table, seq_lens, out, lse=None,
                            scale: float | None = None, stream=None):
    """fa_decode_paged for callers that cannot allocate device memory at decode time.

    The caller passes every buffer, ``out`` included (bf16 or fp32 [S, H, d]; ``lse`` fp32
    [S, H] or None); the split-context scratch is the library's static 32 MiB device array, so
    nothing is allocated here or in the library.  Calls that overlap on the GPU share that array
    and race: serialise them.  Sizes needing more scratch than the array holds raise FaError."""
    lib = load_library()
    f = lib.fa_decode_paged_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, i32, vp, i32, vp, i32, vp, i32, i32, i32, ctypes.c_float, vp]
    f.restype = i32
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _require(t, n)
    _require(block_table, "block_table", torch.int32)
    _require(seq_lens, "seq_lens", torch.int32)
    if q.dim() != 3:
        raise ValueError("q must be [S, H, d]")
    S, H, d = q.shape
    P = k_pool.shape[0]
    if k_pool.shape != (P, H, 16, d) or v_pool.shape != k_pool.shape:
        raise ValueError("k_pool / v_pool must be [num_blocks, H, 16, d]")
    if block_table.dim() != 2 or block_table.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_table must be [S, max_blocks] and seq_lens [S]")
    code = _out_code(out.dtype) if isinstance(out, torch.Tensor) else None
    if code is None:
        raise ValueError("out must be a bf16 or fp32 CUDA tensor")
    _require(out, "out", out.dtype)
    if out.shape != (S, H, d):
        raise ValueError("out must be [S, H, d]")
    if lse is not None:
        _require(lse, "lse", torch.float32)
        if lse.shape != (S, H):
            raise ValueError("lse must be [S, H]")
    for t, n in ((k_pool, "k_pool"), (v_pool, "v_pool"), (block_table, "block_table"),
                 (seq_lens, "seq_lens"), (out, "out")) + (((lse, "lse"),) if lse is not None else ()):
        if t.device != q.device:
            raise ValueError(f"{n} must be on q's device ({q.device})")
    # the library resolves its scratch array, and launches, on the current device
    with torch.cuda.device(q.device):
        st = f(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_table.data_ptr(),
               block_table.shape[1], seq_lens.data_ptr(), P, out.data_ptr(), code,
               lse.data_ptr() if lse is not None else None, S, H, d,
               float(scale) if scale is not None else 0.0, _stream_handle(stream))
    _check(st, "fa_decode_paged_noalloc")
    return out, lse


def selftest_wait_timeout(limit_us: int = 50_000, stream=None) -> int:
    """Launch the bounded-wait self-test and return the device status it leaves (expect 5,
    FA_ERR_TIMEOUT); the status word is read and cleared."""
    lib = load_library()
    f = lib.fa_selftest_wait_timeout
    f.argtypes = [ctypes.c_uint, ctypes.c_void_p]
    f.restype = ctypes.c_int
    _check(f(limit_us, _stream_handle(stream)), "fa_selftest_wait_timeout")
    return device_status(stream)


def probe_ex2_rate(iters: int = 200_000, stream=None) -> tuple[int, float]:
    """Run the exponential-throughput probe once on the current device; returns (exponentials
    launched, device milliseconds from CUDA events on the stream)."""
    lib = load_library()
    f = lib.fa_probe_ex2_rate
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_longlong), ctypes.c_void_p]
    f.restype = ctypes.c_int
    s = stream if stream is not None else torch.cuda.current_stream()
    sink = torch.zeros(1, dtype=torch.float32, device="cuda")
    n = ctypes.c_longlong(0)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    _check(f(sink.data_ptr(), int(iters), ctypes.byref(n), int(s.cuda_stream)), "fa_probe_ex2_rate")
    b.record(s)
    b.synchronize()
    return int(n.value), a.elapsed_time(b)


def probe_read_rate(buf: torch.Tensor, stream=None) -> float:
    """Read every byte of the contiguous CUDA tensor `buf` once with the decode's streaming loads;
    returns the device milliseconds (CUDA events on the stream)."""
    lib = load_library()
    f = lib.fa_probe_read_rate
    f.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    if not buf.is_cuda or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous CUDA tensor")
    s = stream if stream is not None else torch.cuda.current_stream()
    sink = torch.zeros(1, dtype=torch.float32, device=buf.device)
    nbytes = buf.numel() * buf.element_size()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    _check(f(buf.data_ptr(), nbytes, sink.data_ptr(), int(s.cuda_stream)), "fa_probe_read_rate")
    b.record(s)
    b.synchronize()
    return a.elapsed_time(b)


def fwd_schedule(B: int, H: int, N: int, d: int, num_ctas: int):
    """The unit-to-CTA assignment of a causal fa_fwd launch of this shape on `num_ctas` SMs (host
    only).  Returns (start, unit) int32 numpy arrays, CTA c running unit[start[c]:start[c+1]] in
    order, or None when the launch deals its units in snake order instead."""
    import numpy as np
    lib = load_library()
    f = lib.fa_fwd_schedule
    ip = ctypes.POINTER(ctypes.c_int)
    f.argtypes = [ctypes.c_int] * 5 + [ip, ip, ctypes.c_int, ip]
    f.restype = ctypes.c_int
    units = B * H * ((N + 255) // 256)
    start = np.zeros(num_ctas + 1, dtype=np.int32)
    unit = np.zeros(max(units, 1), dtype=np.int32)
    count = ctypes.c_int(0)
    _check(f(B, H, N, d, num_ctas, start.ctypes.data_as(ip), unit.ctypes.data_as(ip), unit.size,
             ctypes.byref(count)), "fa_fwd_schedule")
    return (start, unit[:count.value]) if count.value > 0 else None
