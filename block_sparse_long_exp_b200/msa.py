"""Python binding of libmsa (the C ABI in include/msa.h).

Argument marshalling only: every step of the MSA forward runs in the CUDA
kernels of libmsa.so.  PyTorch provides device memory and streams.  The
functions carry the C entry points' names.  There is no fallback: if the
library is missing or no CUDA device is present, every call raises.

One layer's forward (packed sequences; queries are the last T_b tokens of
each sequence, all tensors bf16 on the GPU except the int32 offsets):

    shape = make_shape(H=64, G=4, d=128, d_idx=64, k=16)        # B_k = 128
    seqs = make_varlen(cu_q, cu_k, cu_q_host, cu_k_host)
    sel = msa_index_topk(shape, seqs, q_idx, k_idx)              # [T, G, k] int32
    out, lse = msa_sparse_attn_prefill(shape, seqs, q, k, v, sel) # [T, H, d], [T, H]

with q [T, H, d], k / v [S, G, d], q_idx [T, G, d_idx], k_idx [S, d_idx].
Decode (one query per sequence) is msa_index_topk + msa_sparse_attn_decode,
or the *_decode_paged pair over a paged cache (make_paged).  Each call
allocates its workspace unless `ws` is given, and by default reads the
device error word afterwards (a synchronisation); pass check=False inside
timed or captured regions and call msa_get_device_error on the workspace
later.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

MSA_OK = 0
STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_WORKSPACE",
          4: "MSA_ERR_CUDA", 5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_DEVICE_CHECK"}

# Every function declared in include/msa.h.
EXPORTED = [
    "msa_index_topk_workspace_size", "msa_index_topk",
    "msa_sparse_attn_workspace_size", "msa_sparse_attn_prefill", "msa_sparse_attn_decode",
    "msa_combine", "msa_dense_attn_workspace_size", "msa_dense_attn",
    "msa_index_topk_decode_noalloc_max_scratch", "msa_index_topk_decode_noalloc",
    "msa_profile_enable", "msa_profile_reset", "msa_profile_read",
    "msa_get_device_error", "msa_version", "msa_set_tile_threshold",
    "msa_decode_paged_workspace_size", "msa_index_topk_decode_paged", "msa_sparse_attn_decode_paged",
]


class MsaError(RuntimeError):
    pass


class Shape(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("G", ctypes.c_int32), ("d", ctypes.c_int32),
                ("d_idx", ctypes.c_int32), ("B_k", ctypes.c_int32), ("k", ctypes.c_int32),
                ("sm_scale", ctypes.c_float)]


class Varlen(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("max_q_len", ctypes.c_int32),
                ("max_k_len", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
                ("cu_q", ctypes.c_void_p), ("cu_k", ctypes.c_void_p)]


class Paged(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("max_blocks", ctypes.c_int32), ("max_seqlen", ctypes.c_int32),
                ("pad_", ctypes.c_int32), ("num_pages", ctypes.c_int64),
                ("seqlens", ctypes.c_void_p), ("block_table", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmsa.so (built by ``block_sparse_long_exp_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise MsaError(f"libmsa.so not found at {path}: build it with "
                       "`python -m block_sparse_long_exp_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
    P = ctypes.POINTER
    lib.msa_index_topk_workspace_size.argtypes = [P(Shape), P(Varlen)]
    lib.msa_index_topk_workspace_size.restype = sz
    lib.msa_index_topk.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, sz, vp]
    lib.msa_index_topk.restype = i32
    lib.msa_sparse_attn_workspace_size.argtypes = [P(Shape), P(Varlen), i64]
    lib.msa_sparse_attn_workspace_size.restype = sz
    lib.msa_sparse_attn_prefill.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp, vp, i64, vp, sz, vp]
    lib.msa_sparse_attn_prefill.restype = i32
    lib.msa_sparse_attn_decode.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_sparse_attn_decode.restype = i32
    lib.msa_combine.argtypes = [P(Shape), i64, vp, vp, vp, vp, vp, vp]
    lib.msa_combine.restype = i32
    lib.msa_dense_attn_workspace_size.argtypes = [P(Shape), P(Varlen)]
    lib.msa_dense_attn_workspace_size.restype = sz
    lib.msa_dense_attn.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_dense_attn.restype = i32
    lib.msa_get_device_error.argtypes = [vp, P(i32), P(i32), P(i32), P(i32), vp]
    lib.msa_get_device_error.restype = i32
    lib.msa_index_topk_decode_noalloc_max_scratch.argtypes = []
    lib.msa_index_topk_decode_noalloc_max_scratch.restype = sz
    lib.msa_index_topk_decode_noalloc.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp]
    lib.msa_index_topk_decode_noalloc.restype = i32
    lib.msa_profile_enable.argtypes = [ctypes.c_int]
    lib.msa_profile_enable.restype = i32
    lib.msa_profile_reset.argtypes = []
    lib.msa_profile_reset.restype = i32
    lib.msa_profile_read.argtypes = [ctypes.c_char_p, P(ctypes.c_double), P(i64)]
    lib.msa_profile_read.restype = i32
    lib.msa_version.argtypes = []
    lib.msa_version.restype = ctypes.c_char_p
    lib.msa_set_tile_threshold.argtypes = [i32]
    lib.msa_set_tile_threshold.restype = i32
    lib.msa_decode_paged_workspace_size.argtypes = [P(Shape), P(Paged)]
    lib.msa_decode_paged_workspace_size.restype = sz
    lib.msa_index_topk_decode_paged.argtypes = [P(Shape), P(Paged), vp, vp, vp, vp, sz, vp]
    lib.msa_index_topk_decode_paged.restype = i32
    lib.msa_sparse_attn_decode_paged.argtypes = [P(Shape), P(Paged), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_sparse_attn_decode_paged.restype = i32
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != MSA_OK:
        raise MsaError(f"{what} failed: {STATUS.get(rc, rc)}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_shape(H: int, G: int, d: int, d_idx: int, k: int, B_k: int = 128,
               sm_scale: Optional[float] = None) -> Shape:
    return Shape(H, G, d, d_idx, B_k, k, float(sm_scale if sm_scale is not None else d ** -0.5))


def make_varlen(cu_q: torch.Tensor, cu_k: torch.Tensor, cu_q_host: Sequence[int],
                cu_k_host: Sequence[int]) -> Varlen:
    """cu_q / cu_k: int32 device tensors [B+1]; the host copies give the sizes."""
    T_lens = [cu_q_host[i + 1] - cu_q_host[i] for i in range(len(cu_q_host) - 1)]
    S_lens = [cu_k_host[i + 1] - cu_k_host[i] for i in range(len(cu_k_host) - 1)]
    return Varlen(len(T_lens), max(T_lens) if T_lens else 0, max(S_lens) if S_lens else 0, 0,
                  int(cu_q_host[-1]), int(cu_k_host[-1]), cu_q.data_ptr(), cu_k.data_ptr())


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _require_cuda(t: torch.Tensor):
    if not t.is_cuda:
        raise MsaError("the MSA kernels need CUDA tensors (no CPU path exists)")


def msa_index_topk(shape: Shape, seqs: Varlen, q_idx: torch.Tensor, k_idx: torch.Tensor,
                   sel: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   stream=None, check: bool = True) -> torch.Tensor:
    """Index branch: scores, block max-pool and top-k with the forced local
    block.  Returns sel [T, G, k] int32: the selected block ids of each
    (query, group), ascending, padded with -1."""
    lib = load_library()
    _require_cuda(q_idx)
    T = seqs.total_q
    if sel is None:
        sel = torch.empty((T, shape.G, shape.k), dtype=torch.int32, device=q_idx.device)
    need = lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(seqs))
    if need == 0:
        raise MsaError("msa_index_topk: unsupported or invalid shape")
    if ws is None:
        ws = _workspace(need, q_idx.device)
    rc = lib.msa_index_topk(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q_idx), _ptr(k_idx), _ptr(sel),
                            _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "msa_index_topk")
    if check:
        _device_check(ws, stream, "msa_index_topk")
    return sel


def msa_index_topk_decode_noalloc(shape: Shape, seqs: Varlen, q_idx: torch.Tensor, k_idx: torch.Tensor,
                                  sel: torch.Tensor, device_error: Optional[torch.Tensor] = None,
                                  stream=None) -> torch.Tensor:
    """Decode-shaped index top-k on the library's fixed scratch array (no
    workspace argument, no allocation inside the call).  `sel` must be given."""
    lib = load_library()
    _require_cuda(q_idx)
    rc = lib.msa_index_topk_decode_noalloc(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q_idx), _ptr(k_idx),
                                           _ptr(sel), _ptr(device_error), _stream(stream))
    _check(rc, "msa_index_topk_decode_noalloc")
    return sel


def msa_index_topk_decode_noalloc_max_scratch() -> int:
    return load_library().msa_index_topk_decode_noalloc_max_scratch()


def msa_sparse_attn_workspace_size(shape: Shape, seqs: Varlen, q_chunk: int = 0) -> int:
    return load_library().msa_sparse_attn_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), q_chunk)


def msa_sparse_attn_prefill(shape: Shape, seqs: Varlen, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            sel: torch.Tensor, out: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None, want_lse: bool = True, q_chunk: int = 0,
                            ws: Optional[torch.Tensor] = None, stream=None,
                            check: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Main branch: exact causal softmax attention of every query over the
    tokens of its selected blocks.  Returns out [T, H, d] bf16 and lse [T, H]
    (natural log; None with want_lse=False).  q_chunk > 0 runs the attention
    in passes of that many query rows (bounded workspace)."""
    lib = load_library()
    _require_cuda(q)
    T = seqs.total_q
    if out is None:
        out = torch.empty((T, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, shape.H), dtype=torch.float32, device=q.device)
    need = msa_sparse_attn_workspace_size(shape, seqs, q_chunk)
    if need == 0:
        raise MsaError("msa_sparse_attn_prefill: unsupported or invalid shape")
    if ws is None:
        ws = _workspace(need, q.device)
    rc = lib.msa_sparse_attn_prefill(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(sel), _ptr(out), _ptr(lse), q_chunk, _ptr(ws), ws.numel(),
                                     _stream(stream))
    _check(rc, "msa_sparse_attn_prefill")
    if check:
        _device_check(ws, stream, "msa_sparse_attn_prefill")
    return out, lse


def msa_sparse_attn_decode(shape: Shape, seqs: Varlen, q: torch.Tensor, k_cache: torch.Tensor,
                           v_cache: torch.Tensor, sel: torch.Tensor, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                           ws: Optional[torch.Tensor] = None, stream=None,
                           check: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Main branch for one query per sequence (its position is the cache's
    last token).  Same outputs as msa_sparse_attn_prefill."""
    lib = load_library()
    _require_cuda(q)
    T = seqs.total_q
    if out is None:
        out = torch.empty((T, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, shape.H), dtype=torch.float32, device=q.device)
    need = msa_sparse_attn_workspace_size(shape, seqs, 0)
    if ws is None:
        ws = _workspace(need, q.device)
    rc = lib.msa_sparse_attn_decode(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k_cache),
                                    _ptr(v_cache), _ptr(sel), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                    _stream(stream))
    _check(rc, "msa_sparse_attn_decode")
    if check:
        _device_check(ws, stream, "msa_sparse_attn_decode")
    return out, lse


def msa_combine(shape: Shape, T: int, part_acc: torch.Tensor, part_lse: torch.Tensor, sel: torch.Tensor,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    lib = load_library()
    _require_cuda(part_acc)
    if out is None:
        out = torch.empty((T, shape.H, shape.d), dtype=torch.bfloat16, device=part_acc.device)
    rc = lib.msa_combine(ctypes.byref(shape), T, _ptr(part_acc), _ptr(part_lse), _ptr(sel), _ptr(out),
                         _ptr(lse), _stream(stream))
    _check(rc, "msa_combine")
    return out, lse


def msa_dense_attn(shape: Shape, seqs: Varlen, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   want_lse: bool = False, ws: Optional[torch.Tensor] = None,
                   stream=None, check: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Dense causal GQA attention (every key at or before the query position)."""
    lib = load_library()
    _require_cuda(q)
    T = seqs.total_q
    if out is None:
        out = torch.empty((T, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, shape.H), dtype=torch.float32, device=q.device)
    need = lib.msa_dense_attn_workspace_size(ctypes.byref(shape), ctypes.byref(seqs))
    if ws is None:
        ws = _workspace(need, q.device)
    rc = lib.msa_dense_attn(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                            _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "msa_dense_attn")
    if check:
        _device_check(ws, stream, "msa_dense_attn")
    return out, lse


def msa_get_device_error(ws: torch.Tensor, stream=None) -> Tuple[int, int, int, int]:
    lib = load_library()
    code, where, i0, i1 = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    rc = lib.msa_get_device_error(_ptr(ws), ctypes.byref(code), ctypes.byref(where), ctypes.byref(i0),
                                  ctypes.byref(i1), _stream(stream))
    _check(rc, "msa_get_device_error")
    return code.value, where.value, i0.value, i1.value


def _device_check(ws: torch.Tensor, stream, what: str):
    code, where, i0, i1 = msa_get_device_error(ws, stream)
    if code != MSA_OK:
        raise MsaError(f"{what}: device reported {STATUS.get(code, code)} at site {where} ({i0}, {i1})")


def msa_profile_enable(on: bool = True):
    _check(load_library().msa_profile_enable(1 if on else 0), "msa_profile_enable")


def msa_profile_reset():
    _check(load_library().msa_profile_reset(), "msa_profile_reset")


def msa_profile_read(kernel: Optional[str]) -> Tuple[float, int]:
    """(total device ms, launches) of one kernel; kernel=None: (0, all launches)."""
    ms, n = ctypes.c_double(), ctypes.c_int64()
    rc = load_library().msa_profile_read(kernel.encode() if kernel else None, ctypes.byref(ms), ctypes.byref(n))
    _check(rc, "msa_profile_read")
    return ms.value, n.value


def make_paged(seqlens: torch.Tensor, block_table: torch.Tensor, max_seqlen: int, num_pages: int) -> Paged:
    """Paged-cache description: seqlens int32 [batch] and block_table int32
    [batch, max_blocks] on the device; max_seqlen >= every seqlens[b]."""
    assert seqlens.dtype == torch.int32 and block_table.dtype == torch.int32 and block_table.dim() == 2
    assert seqlens.is_cuda and block_table.is_cuda and block_table.is_contiguous()
    p = Paged()
    p.batch, p.max_blocks = block_table.shape[0], block_table.shape[1]
    p.max_seqlen, p.num_pages = int(max_seqlen), int(num_pages)
    p.seqlens, p.block_table = seqlens.data_ptr(), block_table.data_ptr()
    p._keep = (seqlens, block_table)
    return p


def _paged_ws(shape: Shape, pages: Paged, ws, device):
    need = load_library().msa_decode_paged_workspace_size(ctypes.byref(shape), ctypes.byref(pages))
    if need == 0:
        raise MsaError("msa_decode_paged_workspace_size: shape or paged description rejected")
    return _workspace(need, device) if ws is None else ws


def msa_index_topk_decode_paged(shape: Shape, pages: Paged, q_idx: torch.Tensor, k_idx_pages: torch.Tensor,
                                sel: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                                stream=None, check: bool = True) -> torch.Tensor:
    lib = load_library()
    _require_cuda(q_idx)
    if sel is None:
        sel = torch.empty((pages.batch, shape.G, shape.k), dtype=torch.int32, device=q_idx.device)
    ws = _paged_ws(shape, pages, ws, q_idx.device)
    rc = lib.msa_index_topk_decode_paged(ctypes.byref(shape), ctypes.byref(pages), _ptr(q_idx), _ptr(k_idx_pages),
                                         _ptr(sel), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "msa_index_topk_decode_paged")
    if check:
        _device_check(ws, stream, "msa_index_topk_decode_paged")
    return sel


def msa_sparse_attn_decode_paged(shape: Shape, pages: Paged, q: torch.Tensor, k_pages: torch.Tensor,
                                 v_pages: torch.Tensor, sel: torch.Tensor, out: Optional[torch.Tensor] = None,
                                 lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                                 ws: Optional[torch.Tensor] = None, stream=None,
                                 check: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    lib = load_library()
    _require_cuda(q)
    if out is None:
        out = torch.empty((pages.batch, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((pages.batch, shape.H), dtype=torch.float32, device=q.device)
    ws = _paged_ws(shape, pages, ws, q.device)
    rc = lib.msa_sparse_attn_decode_paged(ctypes.byref(shape), ctypes.byref(pages), _ptr(q), _ptr(k_pages),
                                          _ptr(v_pages), _ptr(sel), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                          _stream(stream))
    _check(rc, "msa_sparse_attn_decode_paged")
    if check:
        _device_check(ws, stream, "msa_sparse_attn_decode_paged")
    return out, lse


def msa_set_tile_threshold(theta: int) -> int:
    """Query-tile threshold of the prefill main branch (-1 automatic, 0 off);
    returns the previous value."""
    return int(load_library().msa_set_tile_threshold(int(theta)))


def msa_version() -> str:
    return load_library().msa_version().decode()
