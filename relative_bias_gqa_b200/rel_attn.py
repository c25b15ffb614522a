"""ctypes binding of the C ABI in include/rel_attn.h.

Argument marshalling only: every step of the operation runs in the CUDA
library.  Importing this module loads ``librel_attn.so`` and raises
ImportError if it has not been built; there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .build import LIB_PATH

REL_ATTN_OK = 0
REL_ATTN_ERR_INVALID_ARG = -1
REL_ATTN_ERR_WORKSPACE_TOO_SMALL = -2
REL_ATTN_ERR_CUDA = -3
REL_ATTN_ERR_TIMEOUT = -4
REL_ATTN_ERR_BAD_SEQ = -5
REL_ATTN_ERR_NO_DEVICE = -6

EXPORTED = (
    "rel_attn_decode", "rel_attn_partial", "rel_attn_combine", "rel_attn_workspace_bytes", "rel_attn_workspace_init",
    "rel_attn_read_status", "rel_attn_choose_splits", "rel_attn_bucket",
    "rel_attn_error_string", "rel_attn_version", "rel_attn_decode_static",
    "rel_attn_split_pages", "rel_attn_decode_e4m3", "rel_attn_partial_e4m3",
    "rel_attn_set_wait_limit", "rel_attn_kv_write", "rel_attn_prefill",
    "rel_attn_split_pages_e4m3",
)


class RelAttnShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "q_tokens", "num_q_heads", "num_kv_heads", "head_dim",
        "page_size", "num_pages", "max_pages_per_seq", "num_buckets",
        "exact_buckets", "max_distance", "max_seq_len", "out_fp32")]


class RelAttnError(RuntimeError):
    def __init__(self, code: int):
        self.code = code
        super().__init__(f"rel_attn error {code}: {error_string(code)}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m relative_bias_gqa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    SP = ctypes.POINTER(RelAttnShape)
    lib.rel_attn_decode.argtypes = [SP, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                    P, P, P, ctypes.c_size_t, P]
    lib.rel_attn_decode.restype = ctypes.c_int
    lib.rel_attn_partial.argtypes = lib.rel_attn_decode.argtypes
    lib.rel_attn_partial.restype = ctypes.c_int
    lib.rel_attn_combine.argtypes = [SP, ctypes.c_int, P, P, P, ctypes.c_size_t, P]
    lib.rel_attn_combine.restype = ctypes.c_int
    lib.rel_attn_decode_e4m3.argtypes = [SP, P, P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                         P, P, P, ctypes.c_size_t, P]
    lib.rel_attn_decode_e4m3.restype = ctypes.c_int
    lib.rel_attn_partial_e4m3.argtypes = lib.rel_attn_decode_e4m3.argtypes
    lib.rel_attn_partial_e4m3.restype = ctypes.c_int
    lib.rel_attn_decode_static.argtypes = [SP, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                           P, P, P]
    lib.rel_attn_decode_static.restype = ctypes.c_int
    lib.rel_attn_workspace_bytes.argtypes = [SP, ctypes.c_int]
    lib.rel_attn_workspace_bytes.restype = ctypes.c_size_t
    lib.rel_attn_workspace_init.argtypes = [P, ctypes.c_size_t, P]
    lib.rel_attn_workspace_init.restype = ctypes.c_int
    lib.rel_attn_read_status.argtypes = [P, P]
    lib.rel_attn_read_status.restype = ctypes.c_int
    lib.rel_attn_choose_splits.argtypes = [SP, ctypes.c_int, ctypes.c_int]
    lib.rel_attn_choose_splits.restype = ctypes.c_int
    lib.rel_attn_bucket.argtypes = [SP, ctypes.c_int]
    lib.rel_attn_bucket.restype = ctypes.c_int
    lib.rel_attn_split_pages.argtypes = [SP, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.rel_attn_split_pages.restype = ctypes.c_int
    lib.rel_attn_split_pages_e4m3.argtypes = lib.rel_attn_split_pages.argtypes
    lib.rel_attn_split_pages_e4m3.restype = ctypes.c_int
    lib.rel_attn_prefill.argtypes = lib.rel_attn_decode.argtypes
    lib.rel_attn_prefill.restype = ctypes.c_int
    lib.rel_attn_kv_write.argtypes = [SP, P, P, P, P, P, P, P, P, P, P, P, P, P]
    lib.rel_attn_kv_write.restype = ctypes.c_int
    lib.rel_attn_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    lib.rel_attn_set_wait_limit.restype = ctypes.c_int
    lib.rel_attn_error_string.argtypes = [ctypes.c_int]
    lib.rel_attn_error_string.restype = ctypes.c_char_p
    lib.rel_attn_version.argtypes = []
    lib.rel_attn_version.restype = ctypes.c_char_p
    return lib


lib = _load()


def error_string(code: int) -> str:
    return lib.rel_attn_error_string(code).decode()


def version() -> str:
    return lib.rel_attn_version().decode()


def make_shape(*, batch, q_tokens, num_q_heads, num_kv_heads, num_pages,
               max_pages_per_seq, num_buckets, head_dim=128, page_size=64,
               exact_buckets=1024, max_distance=1 << 20, max_seq_len=0,
               out_fp32=False) -> RelAttnShape:
    return RelAttnShape(batch, q_tokens, num_q_heads, num_kv_heads, head_dim,
                        page_size, num_pages, max_pages_per_seq, num_buckets,
                        exact_buckets, max_distance, max_seq_len, int(out_fp32))


def shape_of(q, k_cache, block_table, rel_table, *, max_seq_len=0, out_fp32=False,
             exact_buckets=1024, max_distance=1 << 20) -> RelAttnShape:
    B, T, Hq, D = q.shape
    num_pages, Hkv, P, _ = k_cache.shape
    return make_shape(batch=B, q_tokens=T, num_q_heads=Hq, num_kv_heads=Hkv,
                      num_pages=num_pages, max_pages_per_seq=block_table.shape[1],
                      num_buckets=rel_table.shape[1], head_dim=D, page_size=P,
                      exact_buckets=exact_buckets, max_distance=max_distance,
                      max_seq_len=max_seq_len, out_fp32=out_fp32)


def rel_attn_workspace_bytes(shape: RelAttnShape, num_splits: int = 0) -> int:
    return int(lib.rel_attn_workspace_bytes(ctypes.byref(shape), num_splits))


def rel_attn_choose_splits(shape: RelAttnShape, window: int, sm_count: int = 0) -> int:
    r = lib.rel_attn_choose_splits(ctypes.byref(shape), window, sm_count)
    if r < 0:
        raise RelAttnError(r)
    return r


def rel_attn_bucket(shape: RelAttnShape, distance: int) -> int:
    return int(lib.rel_attn_bucket(ctypes.byref(shape), int(distance)))


def rel_attn_split_pages(shape: RelAttnShape, seq_len: int, window: int, num_splits: int,
                         split: int, e4m3: bool = False):
    """(first_page, end_page) of one split, as the partial kernel (the E4M3
    one with e4m3=True) walks it."""
    a, b = ctypes.c_int(), ctypes.c_int()
    fn = lib.rel_attn_split_pages_e4m3 if e4m3 else lib.rel_attn_split_pages
    rc = fn(ctypes.byref(shape), int(seq_len), int(window), int(num_splits),
            int(split), ctypes.byref(a), ctypes.byref(b))
    if rc != REL_ATTN_OK:
        raise RelAttnError(rc)
    return a.value, b.value


def rel_attn_set_wait_limit(limit_ns: int) -> None:
    """Bound of each device-side wait in later launches (0: the 2 s default)."""
    lib.rel_attn_set_wait_limit(int(limit_ns))


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


class Workspace:
    """Caller-owned device scratch for rel_attn_decode (status word + partials)."""

    def __init__(self, nbytes: int, device):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        rc = lib.rel_attn_workspace_init(ctypes.c_void_p(self.buf.data_ptr()),
                                         self.nbytes, ctypes.c_void_p(_stream_ptr(None)))
        if rc != REL_ATTN_OK:
            raise RelAttnError(rc)

    @classmethod
    def for_shape(cls, shape: RelAttnShape, num_splits: int, device) -> "Workspace":
        n = rel_attn_workspace_bytes(shape, num_splits)
        if n == 0:
            raise RelAttnError(REL_ATTN_ERR_INVALID_ARG)
        return cls(n, device)

    def read_status(self, stream=None) -> int:
        return int(lib.rel_attn_read_status(ctypes.c_void_p(self.buf.data_ptr()),
                                            ctypes.c_void_p(_stream_ptr(stream))))


def rel_attn_decode(q, k_cache, v_cache, block_table, seq_lens, rel_table,
                    window: int = 0, num_splits: int = 0, out=None, lse=None,
                    workspace: Optional[Workspace] = None, *, max_seq_len: int = 0,
                    out_fp32: bool = False, exact_buckets: int = 1024,
                    max_distance: int = 1 << 20, stream=None, with_lse: bool = True):
    """Relative-bias GQA decode attention on the current CUDA device.

    q bf16 [B, T, Hq, D]; k_cache / v_cache bf16 [num_pages, Hkv, P, D];
    block_table int32 [B, max_pages]; seq_lens int32 [B]; rel_table bf16
    [Hkv, NB, D] -- all contiguous CUDA tensors.  Returns (out, lse).
    Supported: D = 128, P = 64, Hq / Hkv in {4, 6, 8} with T <= 9 (T <= 8
    for 8); other shapes raise RelAttnError (REL_ATTN_ERR_INVALID_ARG).
    """
    for name, t, dt in (("q", q, torch.bfloat16), ("k_cache", k_cache, torch.bfloat16),
                        ("v_cache", v_cache, torch.bfloat16), ("rel_table", rel_table, torch.bfloat16),
                        ("block_table", block_table, torch.int32), ("seq_lens", seq_lens, torch.int32)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    shape = shape_of(q, k_cache, block_table, rel_table, max_seq_len=max_seq_len,
                     out_fp32=out_fp32, exact_buckets=exact_buckets,
                     max_distance=max_distance)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    if lse is None and with_lse:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = Workspace.for_shape(shape, num_splits, q.device)
    rc = lib.rel_attn_decode(
        ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        block_table.data_ptr(), seq_lens.data_ptr(), rel_table.data_ptr(),
        int(window), int(num_splits), out.data_ptr(),
        lse.data_ptr() if lse is not None else None,
        workspace.buf.data_ptr(), workspace.nbytes, _stream_ptr(stream))
    if rc != REL_ATTN_OK:
        raise RelAttnError(rc)
    return out, lse


def rel_attn_decode_e4m3(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, rel_table,
                         window: int = 0, num_splits: int = 0, out=None, lse=None,
                         workspace: Optional[Workspace] = None, *, max_seq_len: int = 0,
                         out_fp32: bool = False, exact_buckets: int = 1024,
                         max_distance: int = 1 << 20, stream=None, with_lse: bool = True):
    """rel_attn_decode over an E4M3 KV cache: k_codes / v_codes uint8 (or
    float8_e4m3fn) [num_pages, Hkv, P, D], k_scale / v_scale fp32 [Hkv]."""
    if k_codes.dtype == torch.float8_e4m3fn:
        k_codes = k_codes.view(torch.uint8)
    if v_codes.dtype == torch.float8_e4m3fn:
        v_codes = v_codes.view(torch.uint8)
    for name, t, dt in (("q", q, torch.bfloat16), ("k_codes", k_codes, torch.uint8),
                        ("v_codes", v_codes, torch.uint8), ("k_scale", k_scale, torch.float32),
                        ("v_scale", v_scale, torch.float32), ("rel_table", rel_table, torch.bfloat16),
                        ("block_table", block_table, torch.int32), ("seq_lens", seq_lens, torch.int32)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    shape = shape_of(q, k_codes, block_table, rel_table, max_seq_len=max_seq_len,
                     out_fp32=out_fp32, exact_buckets=exact_buckets, max_distance=max_distance)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    if lse is None and with_lse:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = Workspace.for_shape(shape, num_splits, q.device)
    rc = lib.rel_attn_decode_e4m3(
        ctypes.byref(shape), q.data_ptr(), k_codes.data_ptr(), v_codes.data_ptr(),
        k_scale.data_ptr(), v_scale.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(),
        rel_table.data_ptr(), int(window), int(num_splits), out.data_ptr(),
        lse.data_ptr() if lse is not None else None,
        workspace.buf.data_ptr(), workspace.nbytes, _stream_ptr(stream))
    if rc != REL_ATTN_OK:
        raise RelAttnError(rc)
    return out, lse


def rel_attn_prefill(q, k_cache, v_cache, block_table, seq_lens, rel_table, window: int = 0,
                     num_splits: int = 0, out=None, lse=None, workspace: Optional[Workspace] = None,
                     *, max_seq_len: int = 0, out_fp32: bool = False, exact_buckets: int = 1024,
                     max_distance: int = 1 << 20, stream=None, with_lse: bool = True):
    """Attention for all C query tokens of each sequence (q [B, C, Hq, D],
    token t at position seq_len - C + t, causal); arguments as for
    rel_attn_decode.  Returns (out, lse)."""
    for name, t, dt in (("q", q, torch.bfloat16), ("k_cache", k_cache, torch.bfloat16),
                        ("v_cache", v_cache, torch.bfloat16), ("rel_table", rel_table, torch.bfloat16),
                        ("block_table", block_table, torch.int32), ("seq_lens", seq_lens, torch.int32)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    shape = shape_of(q, k_cache, block_table, rel_table, max_seq_len=max_seq_len,
                     out_fp32=out_fp32, exact_buckets=exact_buckets, max_distance=max_distance)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    if lse is None and with_lse:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    if workspace is None:
        n = prefill_workspace_bytes(shape, num_splits)
        workspace = Workspace(n, q.device)
    rc = lib.rel_attn_prefill(
        ctypes.byref(shape), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        block_table.data_ptr(), seq_lens.data_ptr(), rel_table.data_ptr(),
        int(window), int(num_splits), out.data_ptr(),
        lse.data_ptr() if lse is not None else None,
        workspace.buf.data_ptr(), workspace.nbytes, _stream_ptr(stream))
    if rc != REL_ATTN_OK:
        raise RelAttnError(rc)
    return out, lse


def prefill_workspace_bytes(shape: RelAttnShape, num_splits: int) -> int:
    """Workspace bytes rel_attn_prefill needs: the status word, plus, with
    more than one split, every row's partials (the layout of the decode
    workspace for B * C rows).  num_splits <= 0 assumes up to 256."""
    S = num_splits if num_splits > 0 else 256
    rows = shape.batch * shape.q_tokens * shape.num_q_heads
    if S == 1:
        return 256
    return 256 + (S * rows * 4 + 255) // 256 * 256 + S * rows * 128 * 4


def rel_attn_kv_write(k_new, v_new, conv_w, k_raw, v_raw, k_cache, v_cache, block_table,
                      seq_lens, k_scale=None, v_scale=None, workspace: Optional[Workspace] = None,
                      stream=None):
    """The KV-cache producer step (see include/rel_attn.h): short convolution
    of the T new tokens' K/V (k_new / v_new bf16 [B, T, Hkv, D], taps conv_w
    bf16 [2, Hkv, D, 4]), raw K/V into the sconv cache k_raw / v_raw, the
    convolved K/V into k_cache / v_cache (bf16, or uint8 / float8_e4m3fn
    E4M3 codes with k_scale / v_scale fp32 [Hkv]).  In place; returns None."""
    if k_cache.dtype == torch.float8_e4m3fn:
        k_cache = k_cache.view(torch.uint8)
    if v_cache.dtype == torch.float8_e4m3fn:
        v_cache = v_cache.view(torch.uint8)
    e4m3 = k_scale is not None
    cache_dt = torch.uint8 if e4m3 else torch.bfloat16
    checks = [("k_new", k_new, torch.bfloat16), ("v_new", v_new, torch.bfloat16),
              ("conv_w", conv_w, torch.bfloat16), ("k_raw", k_raw, torch.bfloat16),
              ("v_raw", v_raw, torch.bfloat16), ("k_cache", k_cache, cache_dt),
              ("v_cache", v_cache, cache_dt), ("block_table", block_table, torch.int32),
              ("seq_lens", seq_lens, torch.int32)]
    if e4m3:
        checks += [("k_scale", k_scale, torch.float32), ("v_scale", v_scale, torch.float32)]
    for name, t, dt in checks:
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    B, T, Hkv, D = k_new.shape
    shape = make_shape(batch=B, q_tokens=T, num_q_heads=Hkv, num_kv_heads=Hkv,
                       num_pages=k_cache.shape[0], max_pages_per_seq=block_table.shape[1],
                       num_buckets=1, head_dim=D, page_size=k_cache.shape[2])
    rc = lib.rel_attn_kv_write(
        ctypes.byref(shape), k_new.data_ptr(), v_new.data_ptr(), conv_w.data_ptr(),
        k_raw.data_ptr(), v_raw.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        k_scale.data_ptr() if e4m3 else None, v_scale.data_ptr() if e4m3 else None,
        block_table.data_ptr(), seq_lens.data_ptr(),
        workspace.buf.data_ptr() if workspace is not None else None, _stream_ptr(stream))
    if rc != REL_ATTN_OK:
        raise RelAttnError(rc)


class Prepared:
    """A decode call with every argument marshalled once (shape struct, raw
    pointers, workspace), for callers that issue the same call repeatedly.
    ``decode()`` runs rel_attn_decode; ``partial()`` / ``combine()`` run the
    split-phase pair.  Tensors must stay alive and unmoved while in use."""

    def __init__(self, q, k_cache, v_cache, block_table, seq_lens, rel_table, window=0,
                 num_splits=0, *, out=None, lse=None, max_seq_len=0, out_fp32=False,
                 exact_buckets=1024, max_distance=1 << 20, stream=None, k_scale=None,
                 v_scale=None):
        self.shape = shape_of(q, k_cache, block_table, rel_table, max_seq_len=max_seq_len,
                              out_fp32=out_fp32, exact_buckets=exact_buckets,
                              max_distance=max_distance)
        if num_splits <= 0:
            num_splits = rel_attn_choose_splits(self.shape, window, 0)
        self.num_splits = num_splits
        self.out = out if out is not None else torch.empty(
            q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
        self.lse = lse if lse is not None else torch.empty(q.shape[:3], dtype=torch.float32,
                                                           device=q.device)
        self.workspace = Workspace.for_shape(self.shape, num_splits, q.device)
        self.window = int(window)
        self.stream = stream
        # an E4M3 KV cache (uint8 codes) comes with its per-KV-head scales
        self.e4m3 = k_scale is not None
        if self.e4m3 != (v_scale is not None):
            raise ValueError("k_scale and v_scale go together")
        self._keep = (q, k_cache, v_cache, block_table, seq_lens, rel_table, k_scale, v_scale)
        scales = (k_scale.data_ptr(), v_scale.data_ptr()) if self.e4m3 else ()
        self._args = (q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), *scales,
                      block_table.data_ptr(), seq_lens.data_ptr(), rel_table.data_ptr())

    def _common(self):
        return (ctypes.byref(self.shape), *self._args, self.window, self.num_splits,
                self.out.data_ptr(), self.lse.data_ptr(), self.workspace.buf.data_ptr(),
                self.workspace.nbytes, _stream_ptr(self.stream))

    def decode(self):
        rc = (lib.rel_attn_decode_e4m3 if self.e4m3 else lib.rel_attn_decode)(*self._common())
        if rc != REL_ATTN_OK:
            raise RelAttnError(rc)
        return self.out, self.lse

    def partial(self):
        rc = (lib.rel_attn_partial_e4m3 if self.e4m3 else lib.rel_attn_partial)(*self._common())
        if rc != REL_ATTN_OK:
            raise RelAttnError(rc)

    def combine(self):
        rc = lib.rel_attn_combine(ctypes.byref(self.shape), self.num_splits, self.out.data_ptr(),
                                  self.lse.data_ptr(), self.workspace.buf.data_ptr(),
                                  self.workspace.nbytes, _stream_ptr(self.stream))
        if rc != REL_ATTN_OK:
            raise RelAttnError(rc)
