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

Every call checks its tensors on the host first (dtype, exact shape of the
layout above, row-major contiguity, one CUDA device) and make_varlen checks
the offsets (start at 0, never decrease, T_b <= S_b); a failed check raises
MsaError before anything reaches the GPU, since the C entry points receive
bare pointers and cannot see a buffer's size.
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
    "msa_get_device_error", "msa_version", "msa_set_tile_threshold", "msa_set_attn_window",
    "msa_selftest_wait_timeout_workspace_size", "msa_selftest_wait_timeout",
    "msa_index_topk_decode_candidates", "msa_merge_candidates", "msa_select_block_range",
    "msa_decode_paged_workspace_size", "msa_index_topk_decode_paged", "msa_sparse_attn_decode_paged",
    "msa_index_kl", "msa_index_kl_backward", "msa_select_window", "msa_sparse_attn_backward",
    "msa_selected_share", "msa_index_topk_policy", "msa_gather_pages",
    "msa_prefill_workspace_size", "msa_prefill", "msa_set_prefill_overlap", "msa_index_kl_workspace_size",
    "msa_sparse_attn_backward_workspace_size",
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
    lib.msa_prefill_workspace_size.argtypes = [P(Shape), P(Varlen), i64]
    lib.msa_prefill_workspace_size.restype = sz
    lib.msa_prefill.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp, vp, vp, vp, i64, vp, sz, vp]
    lib.msa_prefill.restype = i32
    lib.msa_set_prefill_overlap.argtypes = [i32]
    lib.msa_set_prefill_overlap.restype = i32
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
    lib.msa_set_attn_window.argtypes = [i32]
    lib.msa_set_attn_window.restype = i32
    lib.msa_index_topk_decode_candidates.argtypes = [P(Shape), P(Varlen), vp, vp, i32, vp, vp, vp, sz, vp]
    lib.msa_index_topk_decode_candidates.restype = i32
    lib.msa_merge_candidates.argtypes = [P(Shape), i32, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_merge_candidates.restype = i32
    lib.msa_select_block_range.argtypes = [P(Shape), i32, vp, vp, vp, vp, vp]
    lib.msa_select_block_range.restype = i32
    lib.msa_selftest_wait_timeout_workspace_size.argtypes = []
    lib.msa_selftest_wait_timeout_workspace_size.restype = sz
    lib.msa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp, sz, vp]
    lib.msa_selftest_wait_timeout.restype = i32
    lib.msa_decode_paged_workspace_size.argtypes = [P(Shape), P(Paged)]
    lib.msa_decode_paged_workspace_size.restype = sz
    lib.msa_index_topk_decode_paged.argtypes = [P(Shape), P(Paged), vp, vp, vp, vp, sz, vp]
    lib.msa_index_topk_decode_paged.restype = i32
    lib.msa_sparse_attn_decode_paged.argtypes = [P(Shape), P(Paged), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.msa_sparse_attn_decode_paged.restype = i32
    lib.msa_index_kl.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, vp, vp, vp, sz,
                                 vp]
    lib.msa_index_kl.restype = i32
    lib.msa_index_kl_workspace_size.argtypes = [P(Shape), P(Varlen), i32]
    lib.msa_index_kl_workspace_size.restype = sz
    lib.msa_sparse_attn_backward_workspace_size.argtypes = [P(Shape), P(Varlen), i32]
    lib.msa_sparse_attn_backward_workspace_size.restype = sz
    lib.msa_index_kl_backward.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, vp,
                                          vp, vp, sz, vp]
    lib.msa_index_kl_backward.restype = i32
    lib.msa_select_window.argtypes = [P(Shape), P(Varlen), i32, vp, vp, sz, vp]
    lib.msa_select_window.restype = i32
    lib.msa_sparse_attn_backward.argtypes = [P(Shape), P(Varlen), vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, sz,
                                             vp]
    lib.msa_sparse_attn_backward.restype = i32
    lib.msa_selected_share.argtypes = [vp, vp, i64, vp, vp]
    lib.msa_selected_share.restype = i32
    lib.msa_index_topk_policy.argtypes = [P(Shape), P(Varlen), i32, i32, vp, vp, vp, vp, sz, vp]
    lib.msa_index_topk_policy.restype = i32
    lib.msa_gather_pages.argtypes = [P(Varlen), vp, i32, i64, i64, vp, vp, vp, sz, vp]
    lib.msa_gather_pages.restype = i32
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
    """cu_q / cu_k: int32 device tensors [B+1]; the host copies give the sizes
    and must hold the same values (they are not read back from the device).
    Checks on the host: both start at 0 and never decrease, T_b <= S_b for
    every sequence, totals fit int32."""
    cu_q_host = [int(x) for x in cu_q_host]
    cu_k_host = [int(x) for x in cu_k_host]
    if len(cu_q_host) < 1 or len(cu_q_host) != len(cu_k_host):
        raise MsaError(f"make_varlen: cu_q_host has {len(cu_q_host)} entries, cu_k_host {len(cu_k_host)} "
                       "(both need batch + 1)")
    if cu_q_host[0] != 0 or cu_k_host[0] != 0:
        raise MsaError("make_varlen: cu_q_host and cu_k_host must start at 0")
    T_lens = [cu_q_host[i + 1] - cu_q_host[i] for i in range(len(cu_q_host) - 1)]
    S_lens = [cu_k_host[i + 1] - cu_k_host[i] for i in range(len(cu_k_host) - 1)]
    for b, (Tb, Sb) in enumerate(zip(T_lens, S_lens)):
        if Tb < 0 or Sb < 0:
            raise MsaError(f"make_varlen: offsets decrease at sequence {b}")
        if Tb > Sb:
            raise MsaError(f"make_varlen: sequence {b} has {Tb} queries but {Sb} keys "
                           "(queries are the last T_b of its tokens)")
    if cu_k_host[-1] >= 2 ** 31 or cu_q_host[-1] >= 2 ** 31:
        raise MsaError("make_varlen: totals beyond int32 offsets")
    B = len(T_lens)
    _arg("cu_q", cu_q, torch.int32, shape=(B + 1,))
    _arg("cu_k", cu_k, torch.int32, shape=(B + 1,))
    _require_cuda(cu_q, cu_k)
    v = Varlen(B, max(T_lens) if T_lens else 0, max(S_lens) if S_lens else 0, 0,
               cu_q_host[-1], cu_k_host[-1], cu_q.data_ptr(), cu_k.data_ptr())
    v._keep = (cu_q, cu_k)
    return v


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _require_cuda(*ts: Optional[torch.Tensor]):
    """Every given tensor lives on one CUDA device (the kernels read them
    through plain device pointers)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise MsaError("the MSA kernels need CUDA tensors (no CPU path exists)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise MsaError(f"tensors on different devices ({dev} and {t.device})")


def _arg(name: str, t, dtype: torch.dtype, shape: Optional[Sequence[int]] = None,
         numel: Optional[int] = None, optional: bool = False):
    """Host check of one tensor argument against the layout the C entry point
    reads: dtype, exact shape (or element count for blocked layouts) and
    row-major contiguity.  Raises MsaError before anything reaches the device."""
    if t is None:
        if optional:
            return
        raise MsaError(f"{name}: a tensor is required")
    if not isinstance(t, torch.Tensor):
        raise MsaError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise MsaError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(int(x) for x in shape):
        raise MsaError(f"{name}: shape {tuple(t.shape)}, expected {tuple(int(x) for x in shape)}")
    if numel is not None and t.numel() != int(numel):
        raise MsaError(f"{name}: {t.numel()} elements, expected {int(numel)}")
    if not t.is_contiguous():
        raise MsaError(f"{name}: must be contiguous (row-major)")


def _ws_arg(ws: Optional[torch.Tensor]):
    if ws is not None and not (isinstance(ws, torch.Tensor) and ws.is_contiguous()):
        raise MsaError("ws: expected a contiguous tensor")


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _groups(shape: Shape) -> int:
    """Heads per group; the C entry points reject the shape if H % G != 0."""
    if shape.G <= 0 or shape.H % shape.G != 0:
        raise MsaError(f"shape: H = {shape.H} is not a multiple of G = {shape.G}")
    return shape.H // shape.G


def msa_index_topk(shape: Shape, seqs: Varlen, q_idx: torch.Tensor, k_idx: torch.Tensor,
                   sel: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   stream=None, check: bool = True) -> torch.Tensor:
    """Index branch: scores, block max-pool and top-k with the forced local
    block.  Returns sel [T, G, k] int32: the selected block ids of each
    (query, group), ascending, padded with -1."""
    lib = load_library()
    T, S = seqs.total_q, seqs.total_k
    _arg("q_idx", q_idx, torch.bfloat16, (T, shape.G, shape.d_idx))
    _arg("k_idx", k_idx, torch.bfloat16, (S, shape.d_idx))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k), optional=True)
    _ws_arg(ws)
    _require_cuda(q_idx, k_idx, sel, ws)
    if sel is None:
        sel = torch.empty((T, shape.G, shape.k), dtype=torch.int32, device=q_idx.device)
    need = lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(seqs))
    if need == 0:
        raise MsaError("msa_index_topk: unsupported or invalid shape")
    if ws is None:
        ws = _workspace(need, q_idx.device)
    rc = lib.msa_index_topk(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q_idx), _ptr(k_idx), _ptr(sel),
                            _ptr(ws), _nbytes(ws), _stream(stream))
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
    T, S = seqs.total_q, seqs.total_k
    _arg("q_idx", q_idx, torch.bfloat16, (T, shape.G, shape.d_idx))
    _arg("k_idx", k_idx, torch.bfloat16, (S, shape.d_idx))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k))
    if device_error is not None:
        _arg("device_error", device_error, torch.int32)
        if device_error.numel() < 1:
            raise MsaError("device_error: needs one int32 element")
    _require_cuda(q_idx, k_idx, sel, device_error)
    rc = lib.msa_index_topk_decode_noalloc(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q_idx), _ptr(k_idx),
                                           _ptr(sel), _ptr(device_error), _stream(stream))
    _check(rc, "msa_index_topk_decode_noalloc")
    return sel


def msa_index_topk_decode_noalloc_max_scratch() -> int:
    return load_library().msa_index_topk_decode_noalloc_max_scratch()


def msa_index_topk_workspace_size(shape: Shape, seqs: Varlen) -> int:
    """Workspace bytes msa_index_topk needs (0: shape or sizes unsupported)."""
    return load_library().msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(seqs))


def msa_sparse_attn_workspace_size(shape: Shape, seqs: Varlen, q_chunk: int = 0) -> int:
    """Workspace bytes of the main-branch calls (0: unsupported)."""
    return load_library().msa_sparse_attn_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), q_chunk)


def msa_dense_attn_workspace_size(shape: Shape, seqs: Varlen) -> int:
    """Workspace bytes msa_dense_attn needs (0: unsupported)."""
    return load_library().msa_dense_attn_workspace_size(ctypes.byref(shape), ctypes.byref(seqs))


def msa_decode_paged_workspace_size(shape: Shape, pages: Paged) -> int:
    """Workspace bytes of either paged decode call (0: rejected)."""
    return load_library().msa_decode_paged_workspace_size(ctypes.byref(shape), ctypes.byref(pages))


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
    T, S = seqs.total_q, seqs.total_k
    _arg("q", q, torch.bfloat16, (T, shape.H, shape.d))
    _arg("k", k, torch.bfloat16, (S, shape.G, shape.d))
    _arg("v", v, torch.bfloat16, (S, shape.G, shape.d))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k))
    _arg("out", out, torch.bfloat16, (T, shape.H, shape.d), optional=True)
    _arg("lse", lse, torch.float32, (T, shape.H), optional=True)
    _ws_arg(ws)
    _require_cuda(q, k, v, sel, out, lse, ws)
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
                                     _ptr(sel), _ptr(out), _ptr(lse), q_chunk, _ptr(ws), _nbytes(ws),
                                     _stream(stream))
    _check(rc, "msa_sparse_attn_prefill")
    if check:
        _device_check(ws, stream, "msa_sparse_attn_prefill")
    return out, lse


def msa_prefill_workspace_size(shape: Shape, seqs: Varlen, q_chunk: int = 0) -> int:
    """Workspace bytes of msa_prefill (0: unsupported)."""
    return load_library().msa_prefill_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), q_chunk)


def msa_prefill(shape: Shape, seqs: Varlen, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                q_idx: torch.Tensor, k_idx: torch.Tensor, sel: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                q_chunk: int = 0, ws: Optional[torch.Tensor] = None, stream=None,
                check: bool = True) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """One MSA layer, prefill: index top-k and the main branch in passes of
    q_chunk query rows (the combine of a pass overlaps the next pass's index
    top-k).  Returns sel [T, G, k], out [T, H, d] and lse [T, H] (None with
    want_lse=False), equal to msa_index_topk followed by
    msa_sparse_attn_prefill with the same q_chunk."""
    lib = load_library()
    T, S = seqs.total_q, seqs.total_k
    _arg("q", q, torch.bfloat16, (T, shape.H, shape.d))
    _arg("k", k, torch.bfloat16, (S, shape.G, shape.d))
    _arg("v", v, torch.bfloat16, (S, shape.G, shape.d))
    _arg("q_idx", q_idx, torch.bfloat16, (T, shape.G, shape.d_idx))
    _arg("k_idx", k_idx, torch.bfloat16, (S, shape.d_idx))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k), optional=True)
    _arg("out", out, torch.bfloat16, (T, shape.H, shape.d), optional=True)
    _arg("lse", lse, torch.float32, (T, shape.H), optional=True)
    _ws_arg(ws)
    _require_cuda(q, k, v, q_idx, k_idx, sel, out, lse, ws)
    if sel is None:
        sel = torch.empty((T, shape.G, shape.k), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty((T, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, shape.H), dtype=torch.float32, device=q.device)
    need = msa_prefill_workspace_size(shape, seqs, q_chunk)
    if need == 0:
        raise MsaError("msa_prefill: unsupported or invalid shape")
    if ws is None:
        ws = _workspace(need, q.device)
    rc = lib.msa_prefill(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx),
                         _ptr(k_idx), _ptr(sel), _ptr(out), _ptr(lse), q_chunk, _ptr(ws), _nbytes(ws),
                         _stream(stream))
    _check(rc, "msa_prefill")
    if check:
        _device_check(ws, stream, "msa_prefill")
    return sel, out, lse


def msa_set_prefill_overlap(sms: int) -> int:
    """SMs msa_prefill gives a pass's combine while the next pass's index
    top-k runs (< 0: the default, 0: no overlap); returns the previous value."""
    return int(load_library().msa_set_prefill_overlap(int(sms)))


def msa_sparse_attn_decode(shape: Shape, seqs: Varlen, q: torch.Tensor, k_cache: torch.Tensor,
                           v_cache: torch.Tensor, sel: torch.Tensor, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                           ws: Optional[torch.Tensor] = None, stream=None,
                           check: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Main branch for one query per sequence (its position is the cache's
    last token).  Same outputs as msa_sparse_attn_prefill."""
    lib = load_library()
    T, S = seqs.total_q, seqs.total_k
    _arg("q", q, torch.bfloat16, (T, shape.H, shape.d))
    _arg("k_cache", k_cache, torch.bfloat16, (S, shape.G, shape.d))
    _arg("v_cache", v_cache, torch.bfloat16, (S, shape.G, shape.d))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k))
    _arg("out", out, torch.bfloat16, (T, shape.H, shape.d), optional=True)
    _arg("lse", lse, torch.float32, (T, shape.H), optional=True)
    _ws_arg(ws)
    _require_cuda(q, k_cache, v_cache, sel, out, lse, ws)
    if out is None:
        out = torch.empty((T, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, shape.H), dtype=torch.float32, device=q.device)
    need = msa_sparse_attn_workspace_size(shape, seqs, 0)
    if ws is None:
        ws = _workspace(need, q.device)
    rc = lib.msa_sparse_attn_decode(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k_cache),
                                    _ptr(v_cache), _ptr(sel), _ptr(out), _ptr(lse), _ptr(ws), _nbytes(ws),
                                    _stream(stream))
    _check(rc, "msa_sparse_attn_decode")
    if check:
        _device_check(ws, stream, "msa_sparse_attn_decode")
    return out, lse


def msa_combine(shape: Shape, T: int, part_acc: torch.Tensor, part_lse: torch.Tensor, sel: torch.Tensor,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Log-sum-exp merge of per-block partials: part_acc f16 [T, G, k, d/8, H/G, 8],
    part_lse f32 [T, G, k, H/G], sel int32 [T, G, k] (slots with sel < 0 unused)."""
    lib = load_library()
    Hg = _groups(shape)
    _arg("part_acc", part_acc, torch.float16, numel=T * shape.G * shape.k * Hg * shape.d)
    _arg("part_lse", part_lse, torch.float32, numel=T * shape.G * shape.k * Hg)
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k))
    _arg("out", out, torch.bfloat16, (T, shape.H, shape.d), optional=True)
    _arg("lse", lse, torch.float32, (T, shape.H), optional=True)
    _require_cuda(part_acc, part_lse, sel, out, lse)
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
    T, S = seqs.total_q, seqs.total_k
    _arg("q", q, torch.bfloat16, (T, shape.H, shape.d))
    _arg("k", k, torch.bfloat16, (S, shape.G, shape.d))
    _arg("v", v, torch.bfloat16, (S, shape.G, shape.d))
    _arg("out", out, torch.bfloat16, (T, shape.H, shape.d), optional=True)
    _arg("lse", lse, torch.float32, (T, shape.H), optional=True)
    _ws_arg(ws)
    _require_cuda(q, k, v, out, lse, ws)
    if out is None:
        out = torch.empty((T, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, shape.H), dtype=torch.float32, device=q.device)
    need = lib.msa_dense_attn_workspace_size(ctypes.byref(shape), ctypes.byref(seqs))
    if ws is None:
        ws = _workspace(need, q.device)
    rc = lib.msa_dense_attn(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                            _ptr(lse), _ptr(ws), _nbytes(ws), _stream(stream))
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
    if not isinstance(block_table, torch.Tensor) or block_table.dim() != 2:
        raise MsaError("block_table: expected a 2-D int32 tensor [batch, max_blocks]")
    _arg("block_table", block_table, torch.int32)
    _arg("seqlens", seqlens, torch.int32, (block_table.shape[0],))
    if int(num_pages) < 0 or int(max_seqlen) < 0:
        raise MsaError("make_paged: num_pages and max_seqlen must be >= 0")
    _require_cuda(seqlens, block_table)
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
    """Index branch of one query per sequence over a paged cache: q_idx bf16
    [batch, G, d_idx], k_idx_pages bf16 [num_pages * B_k, d_idx]; returns sel
    int32 [batch, G, k]."""
    lib = load_library()
    B, rows = pages.batch, pages.num_pages * shape.B_k
    _arg("q_idx", q_idx, torch.bfloat16, (B, shape.G, shape.d_idx))
    _arg("k_idx_pages", k_idx_pages, torch.bfloat16, (rows, shape.d_idx))
    _arg("sel", sel, torch.int32, (B, shape.G, shape.k), optional=True)
    _ws_arg(ws)
    _require_cuda(q_idx, k_idx_pages, sel, ws)
    if sel is None:
        sel = torch.empty((pages.batch, shape.G, shape.k), dtype=torch.int32, device=q_idx.device)
    ws = _paged_ws(shape, pages, ws, q_idx.device)
    rc = lib.msa_index_topk_decode_paged(ctypes.byref(shape), ctypes.byref(pages), _ptr(q_idx), _ptr(k_idx_pages),
                                         _ptr(sel), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(rc, "msa_index_topk_decode_paged")
    if check:
        _device_check(ws, stream, "msa_index_topk_decode_paged")
    return sel


def msa_sparse_attn_decode_paged(shape: Shape, pages: Paged, q: torch.Tensor, k_pages: torch.Tensor,
                                 v_pages: torch.Tensor, sel: torch.Tensor, out: Optional[torch.Tensor] = None,
                                 lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                                 ws: Optional[torch.Tensor] = None, stream=None,
                                 check: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Main branch of one query per sequence over paged K / V: q bf16 [batch, H, d],
    k_pages / v_pages bf16 [num_pages * B_k, G, d], sel int32 [batch, G, k];
    returns out bf16 [batch, H, d] and lse f32 [batch, H]."""
    lib = load_library()
    B, rows = pages.batch, pages.num_pages * shape.B_k
    _arg("q", q, torch.bfloat16, (B, shape.H, shape.d))
    _arg("k_pages", k_pages, torch.bfloat16, (rows, shape.G, shape.d))
    _arg("v_pages", v_pages, torch.bfloat16, (rows, shape.G, shape.d))
    _arg("sel", sel, torch.int32, (B, shape.G, shape.k))
    _arg("out", out, torch.bfloat16, (B, shape.H, shape.d), optional=True)
    _arg("lse", lse, torch.float32, (B, shape.H), optional=True)
    _ws_arg(ws)
    _require_cuda(q, k_pages, v_pages, sel, out, lse, ws)
    if out is None:
        out = torch.empty((pages.batch, shape.H, shape.d), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((pages.batch, shape.H), dtype=torch.float32, device=q.device)
    ws = _paged_ws(shape, pages, ws, q.device)
    rc = lib.msa_sparse_attn_decode_paged(ctypes.byref(shape), ctypes.byref(pages), _ptr(q), _ptr(k_pages),
                                          _ptr(v_pages), _ptr(sel), _ptr(out), _ptr(lse), _ptr(ws), _nbytes(ws),
                                          _stream(stream))
    _check(rc, "msa_sparse_attn_decode_paged")
    if check:
        _device_check(ws, stream, "msa_sparse_attn_decode_paged")
    return out, lse


def _index_kl_args(shape, seqs, q, k, q_idx, k_idx, sel, lse, dense):
    T, S = seqs.total_q, seqs.total_k
    _arg("q", q, torch.bfloat16, (T, shape.H, shape.d))
    _arg("k", k, torch.bfloat16, (S, shape.G, shape.d))
    _arg("q_idx", q_idx, torch.bfloat16, (T, shape.G, shape.d_idx))
    _arg("k_idx", k_idx, torch.bfloat16, (S, shape.d_idx))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k), optional=dense)
    _arg("lse", lse, torch.float32, (T, shape.H))


def msa_index_kl_workspace_size(shape: Shape, seqs: Varlen, dense: bool = False) -> int:
    """Workspace bytes of msa_index_kl (0: unsupported)."""
    return load_library().msa_index_kl_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), 1 if dense else 0)


def msa_index_kl(shape: Shape, seqs: Varlen, q: torch.Tensor, k: torch.Tensor, q_idx: torch.Tensor,
                 k_idx: torch.Tensor, sel: Optional[torch.Tensor], lse: torch.Tensor, tau: float,
                 dense: bool = False, kl: Optional[torch.Tensor] = None, want_lse_z: bool = False,
                 ws: Optional[torch.Tensor] = None, stream=None, check: bool = True):
    """Index-alignment target: KL(P || Q) per (query, group) over the support
    (the selected tokens, or with dense=True every token up to the query).
    P: the main branch's attention on the support, averaged over the group's
    heads (lse [T, H] float: its log-sum-exp over that support, as the prefill
    or dense call returns it); Q: softmax of tau * index score.  Returns kl
    float [T, G], or (kl, lse_z) with want_lse_z (the student's log-sum-exp,
    which msa_index_kl_backward takes)."""
    lib = load_library()
    T = seqs.total_q
    _index_kl_args(shape, seqs, q, k, q_idx, k_idx, sel, lse, dense)
    _arg("kl", kl, torch.float32, (T, shape.G), optional=True)
    _ws_arg(ws)
    _require_cuda(q, k, q_idx, k_idx, sel, lse, kl, ws)
    if kl is None:
        kl = torch.empty((T, shape.G), dtype=torch.float32, device=q.device)
    lse_z = torch.empty((T, shape.G), dtype=torch.float32, device=q.device) if want_lse_z else None
    if ws is None:
        need = msa_index_kl_workspace_size(shape, seqs, dense)
        if need == 0:
            raise MsaError("msa_index_kl: unsupported or invalid shape")
        ws = _workspace(need, q.device)
    rc = lib.msa_index_kl(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k), _ptr(q_idx), _ptr(k_idx),
                          _ptr(sel), _ptr(lse), float(tau), 1 if dense else 0, _ptr(kl), _ptr(lse_z), _ptr(ws),
                          _nbytes(ws), _stream(stream))
    _check(rc, "msa_index_kl")
    if check:
        _device_check(ws, stream, "msa_index_kl")
    return (kl, lse_z) if want_lse_z else kl


def msa_index_kl_backward(shape: Shape, seqs: Varlen, q: torch.Tensor, k: torch.Tensor, q_idx: torch.Tensor,
                          k_idx: torch.Tensor, sel: Optional[torch.Tensor], lse: torch.Tensor, lse_z: torch.Tensor,
                          tau: float, dense: bool = False, ws: Optional[torch.Tensor] = None, stream=None,
                          check: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """Gradient of the summed KL with respect to the index query and keys, the
    teacher held constant: returns dq_idx float [T, G, d_idx] and dk_idx float
    [S, d_idx].  lse_z: from msa_index_kl(..., want_lse_z=True).  ws: as
    msa_index_kl's (msa_index_kl_workspace_size bytes)."""
    lib = load_library()
    T, S = seqs.total_q, seqs.total_k
    _index_kl_args(shape, seqs, q, k, q_idx, k_idx, sel, lse, dense)
    _arg("lse_z", lse_z, torch.float32, (T, shape.G))
    _ws_arg(ws)
    _require_cuda(q, k, q_idx, k_idx, sel, lse, lse_z, ws)
    dq = torch.empty((T, shape.G, shape.d_idx), dtype=torch.float32, device=q.device)
    dk = torch.empty((S, shape.d_idx), dtype=torch.float32, device=q.device)
    if ws is None:
        need = msa_index_kl_workspace_size(shape, seqs, dense)
        if need == 0:
            raise MsaError("msa_index_kl_backward: unsupported or invalid shape")
        ws = _workspace(need, q.device)
    rc = lib.msa_index_kl_backward(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k), _ptr(q_idx),
                                   _ptr(k_idx), _ptr(sel), _ptr(lse), _ptr(lse_z), float(tau), 1 if dense else 0,
                                   _ptr(dq), _ptr(dk), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(rc, "msa_index_kl_backward")
    if check:
        _device_check(ws, stream, "msa_index_kl_backward")
    return dq, dk


def msa_select_window(shape: Shape, seqs: Varlen, n_sink: int = 1, sel: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None, device=None, stream=None, check: bool = True) -> torch.Tensor:
    """The FLOP-matched sliding-window baseline's selection: the first n_sink
    blocks and the k - n_sink most recent ones per (query, group), in
    msa_index_topk's layout (sel int32 [T, G, k]), for the main-branch calls."""
    lib = load_library()
    T = seqs.total_q
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k), optional=True)
    _ws_arg(ws)
    dev = sel.device if sel is not None else (device or torch.device("cuda"))
    if sel is None:
        sel = torch.empty((T, shape.G, shape.k), dtype=torch.int32, device=dev)
    _require_cuda(sel, ws)
    if ws is None:
        ws = _workspace(256, sel.device)
    rc = lib.msa_select_window(ctypes.byref(shape), ctypes.byref(seqs), int(n_sink), _ptr(sel), _ptr(ws),
                               _nbytes(ws), _stream(stream))
    _check(rc, "msa_select_window")
    if check:
        _device_check(ws, stream, "msa_select_window")
    return sel


def msa_sparse_attn_backward_workspace_size(shape: Shape, seqs: Varlen, dense: bool = False) -> int:
    """Bytes of workspace msa_sparse_attn_backward takes (0: unsupported shape)."""
    return load_library().msa_sparse_attn_backward_workspace_size(ctypes.byref(shape), ctypes.byref(seqs),
                                                                   1 if dense else 0)


def msa_sparse_attn_backward(shape: Shape, seqs: Varlen, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                             sel: Optional[torch.Tensor], out: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
                             dense: bool = False, ws: Optional[torch.Tensor] = None, stream=None,
                             check: bool = True) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Main Branch backward over the support (the selected tokens, or with
    dense=True every token up to the query): returns dq float [T, H, d] and
    dk, dv float [S, G, d].  out / lse: the forward's outputs for the same
    support; dout: bf16 [T, H, d].  ws: msa_sparse_attn_backward_workspace_size
    bytes (the selected support plans the forward's KV-outer lists there)."""
    lib = load_library()
    T, S = seqs.total_q, seqs.total_k
    _arg("q", q, torch.bfloat16, (T, shape.H, shape.d))
    _arg("k", k, torch.bfloat16, (S, shape.G, shape.d))
    _arg("v", v, torch.bfloat16, (S, shape.G, shape.d))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k), optional=dense)
    _arg("out", out, torch.bfloat16, (T, shape.H, shape.d))
    _arg("lse", lse, torch.float32, (T, shape.H))
    _arg("dout", dout, torch.bfloat16, (T, shape.H, shape.d))
    _ws_arg(ws)
    _require_cuda(q, k, v, sel, out, lse, dout, ws)
    dq = torch.empty((T, shape.H, shape.d), dtype=torch.float32, device=q.device)
    dk = torch.empty((S, shape.G, shape.d), dtype=torch.float32, device=q.device)
    dv = torch.empty((S, shape.G, shape.d), dtype=torch.float32, device=q.device)
    if ws is None:
        need = msa_sparse_attn_backward_workspace_size(shape, seqs, dense)
        if need == 0:
            raise MsaError("msa_sparse_attn_backward: unsupported or invalid shape")
        ws = _workspace(need, q.device)
    rc = lib.msa_sparse_attn_backward(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q), _ptr(k), _ptr(v), _ptr(sel),
                                      _ptr(out), _ptr(lse), _ptr(dout), 1 if dense else 0, _ptr(dq), _ptr(dk),
                                      _ptr(dv), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(rc, "msa_sparse_attn_backward")
    if check:
        _device_check(ws, stream, "msa_sparse_attn_backward")
    return dq, dk, dv


def msa_index_topk_policy(shape: Shape, seqs: Varlen, q_idx: torch.Tensor, k_idx: torch.Tensor, n_sink: int = 1,
                          n_local: int = 1, sel: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                          stream=None, check: bool = True) -> torch.Tensor:
    """Index Branch with n_sink forced first blocks and an n_local-block forced
    local window, the rest of the k blocks by score; sel int32 [T, G, k] as
    msa_index_topk (n_sink=0, n_local=1 is its rule)."""
    lib = load_library()
    T, S = seqs.total_q, seqs.total_k
    _arg("q_idx", q_idx, torch.bfloat16, (T, shape.G, shape.d_idx))
    _arg("k_idx", k_idx, torch.bfloat16, (S, shape.d_idx))
    _arg("sel", sel, torch.int32, (T, shape.G, shape.k), optional=True)
    _ws_arg(ws)
    _require_cuda(q_idx, k_idx, sel, ws)
    if sel is None:
        sel = torch.empty((T, shape.G, shape.k), dtype=torch.int32, device=q_idx.device)
    if ws is None:
        ws = _workspace(256, q_idx.device)
    rc = lib.msa_index_topk_policy(ctypes.byref(shape), ctypes.byref(seqs), int(n_sink), int(n_local), _ptr(q_idx),
                                   _ptr(k_idx), _ptr(sel), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(rc, "msa_index_topk_policy")
    if check:
        _device_check(ws, stream, "msa_index_topk_policy")
    return sel


def _table_arg(seqs: Varlen, block_table: torch.Tensor) -> int:
    """Checks a block table [batch, max_blocks] int32; returns max_blocks."""
    if not isinstance(block_table, torch.Tensor) or block_table.dim() != 2:
        raise MsaError("block_table: expected a 2-D int32 tensor [batch, max_blocks]")
    _arg("block_table", block_table, torch.int32)
    if block_table.shape[0] != seqs.batch:
        raise MsaError(f"block_table: {block_table.shape[0]} rows for {seqs.batch} sequences")
    return int(block_table.shape[1])


def msa_gather_pages(seqs: Varlen, block_table: torch.Tensor, num_pages: int, pages: torch.Tensor,
                     ws: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> torch.Tensor:
    """Rows of a paged cache (pages [num_pages * B_k, ...]) gathered into packed
    rows [total_k, ...] of the sequences seqs describes (cu_k: lengths)."""
    lib = load_library()
    max_blocks = _table_arg(seqs, block_table)
    if not isinstance(pages, torch.Tensor) or pages.dim() < 1 or pages.shape[0] != int(num_pages) * 128:
        raise MsaError("pages: expected a tensor of num_pages * 128 rows")
    _arg("pages", pages, pages.dtype)
    row_bytes = pages[0].numel() * pages.element_size() if pages.shape[0] else 0
    packed = torch.empty((seqs.total_k,) + tuple(pages.shape[1:]), dtype=pages.dtype, device=pages.device)
    _ws_arg(ws)
    _require_cuda(block_table, pages, ws)
    if ws is None:
        ws = _workspace(256, pages.device)
    rc = lib.msa_gather_pages(ctypes.byref(seqs), _ptr(block_table), max_blocks, int(num_pages), int(row_bytes),
                              _ptr(pages), _ptr(packed), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(rc, "msa_gather_pages")
    if check:
        _device_check(ws, stream, "msa_gather_pages")
    return packed


def msa_prefill_paged(shape: Shape, seqs: Varlen, block_table: torch.Tensor, num_pages: int, q: torch.Tensor,
                      q_idx: torch.Tensor, k_idx_pages: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                      q_chunk: int = 0, stream=None):
    """A prefill (or a chunk of one) over a paged cache: the pages gathered into
    packed rows, then msa_index_topk and msa_sparse_attn_prefill.  Returns
    (sel, out, lse)."""
    k_idx = msa_gather_pages(seqs, block_table, num_pages, k_idx_pages, stream=stream)
    k = msa_gather_pages(seqs, block_table, num_pages, k_pages, stream=stream)
    v = msa_gather_pages(seqs, block_table, num_pages, v_pages, stream=stream)
    sel = msa_index_topk(shape, seqs, q_idx, k_idx, stream=stream)
    out, lse = msa_sparse_attn_prefill(shape, seqs, q, k, v, sel, q_chunk=q_chunk, stream=stream)
    return sel, out, lse


def msa_selected_share(lse_sel: torch.Tensor, lse_all: torch.Tensor, stream=None) -> torch.Tensor:
    """Share of each head's dense causal attention weight on the selected
    tokens: exp(lse_sel - lse_all), lse_sel from msa_sparse_attn_prefill and
    lse_all from msa_dense_attn (float [T, H] each)."""
    lib = load_library()
    _arg("lse_sel", lse_sel, torch.float32)
    _arg("lse_all", lse_all, torch.float32, tuple(lse_sel.shape))
    _require_cuda(lse_sel, lse_all)
    share = torch.empty_like(lse_sel)
    rc = lib.msa_selected_share(_ptr(lse_sel), _ptr(lse_all), lse_sel.numel(), _ptr(share), _stream(stream))
    _check(rc, "msa_selected_share")
    return share


def msa_set_tile_threshold(theta: int) -> int:
    """Query-tile threshold of the prefill main branch (-1 automatic, 0 off);
    returns the previous value."""
    return int(load_library().msa_set_tile_threshold(int(theta)))


def msa_index_topk_decode_candidates(shape: Shape, seqs: Varlen, q_idx: torch.Tensor, k_idx: torch.Tensor,
                                     all_blocks: bool, ws: Optional[torch.Tensor] = None, stream=None,
                                     check: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per (query, group) the k-1 best blocks of a key slice and their scores
    (decode shape; ids local to the slice, -1 / -inf padding): the candidates
    of one rank of a key-range split (see msa_merge_candidates)."""
    lib = load_library()
    G, kc = shape.G, max(shape.k - 1, 0)
    T = int(seqs.total_q)
    _arg("q_idx", q_idx, torch.bfloat16, (T, G, shape.d_idx))
    _arg("k_idx", k_idx, torch.bfloat16, (int(seqs.total_k), shape.d_idx))
    _require_cuda(q_idx, k_idx)
    ids = torch.full((T, G, kc), -1, dtype=torch.int32, device=q_idx.device)
    scores = torch.full((T, G, kc), float("-inf"), dtype=torch.float32, device=q_idx.device)
    if ws is None:
        ws = _workspace(lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(seqs)), q_idx.device)
    _ws_arg(ws)
    rc = lib.msa_index_topk_decode_candidates(ctypes.byref(shape), ctypes.byref(seqs), _ptr(q_idx), _ptr(k_idx),
                                              int(bool(all_blocks)), _ptr(ids), _ptr(scores), _ptr(ws), _nbytes(ws),
                                              _stream(stream))
    _check(rc, "msa_index_topk_decode_candidates")
    if check:
        _device_check(ws, stream, "msa_index_topk_decode_candidates")
    return ids, scores


def msa_merge_candidates(shape: Shape, cand_ids: torch.Tensor, cand_scores: torch.Tensor,
                         local_block: torch.Tensor, stream=None, check: bool = True) -> torch.Tensor:
    """The selection of a key-range split: the top k-1 of the candidates
    [batch, G, n_cand] (global block ids) in the selection order, with the
    local block [batch] forced; sel [batch, G, k] as msa_index_topk writes it."""
    lib = load_library()
    G = shape.G
    _arg("cand_ids", cand_ids, torch.int32)
    if cand_ids.dim() != 3 or cand_ids.shape[1] != G:
        raise MsaError(f"cand_ids: expected [batch, {G}, n_cand], got {tuple(cand_ids.shape)}")
    B, _, n = cand_ids.shape
    _arg("cand_scores", cand_scores, torch.float32, (B, G, n))
    _arg("local_block", local_block, torch.int32, (B,))
    _require_cuda(cand_ids, cand_scores, local_block)
    sel = torch.empty((B, G, shape.k), dtype=torch.int32, device=cand_ids.device)
    ws = _workspace(256, cand_ids.device)
    rc = lib.msa_merge_candidates(ctypes.byref(shape), B, n, _ptr(cand_ids), _ptr(cand_scores), _ptr(local_block),
                                  _ptr(sel), _ptr(ws), _nbytes(ws), _stream(stream))
    _check(rc, "msa_merge_candidates")
    if check:
        _device_check(ws, stream, "msa_merge_candidates")
    return sel


def msa_select_block_range(shape: Shape, sel: torch.Tensor, blk_lo: torch.Tensor, blk_hi: torch.Tensor,
                           stream=None) -> torch.Tensor:
    """The blocks of a selection [batch, G, k] inside [blk_lo[b], blk_hi[b]),
    re-based to the range, ascending, -1 padded."""
    lib = load_library()
    G = shape.G
    _arg("sel", sel, torch.int32)
    if sel.dim() != 3 or sel.shape[1:] != (G, shape.k):
        raise MsaError(f"sel: expected [batch, {G}, {shape.k}], got {tuple(sel.shape)}")
    B = sel.shape[0]
    _arg("blk_lo", blk_lo, torch.int32, (B,))
    _arg("blk_hi", blk_hi, torch.int32, (B,))
    _require_cuda(sel, blk_lo, blk_hi)
    out = torch.empty_like(sel)
    rc = lib.msa_select_block_range(ctypes.byref(shape), B, _ptr(sel), _ptr(blk_lo), _ptr(blk_hi), _ptr(out),
                                    _stream(stream))
    _check(rc, "msa_select_block_range")
    return out


def msa_selftest_wait_timeout(limit_us: int = 2000, stream=None) -> Tuple[int, int, int, int]:
    """Run the bounded-wait self-test (two waits that nothing ever ends, each
    with a `limit_us` limit) and return (error code, site, waits that ran out,
    0) once the stream has drained."""
    lib = load_library()
    n = int(lib.msa_selftest_wait_timeout_workspace_size())
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    _check(lib.msa_selftest_wait_timeout(int(limit_us), _ptr(ws), n, _stream(stream)), "msa_selftest_wait_timeout")
    code, where, _, _ = msa_get_device_error(ws, stream)
    timed_out = int(ws[260:264].view(torch.int32).item())
    return code, where, timed_out, 0


def msa_set_attn_window(rows: int) -> int:
    """Query rows per planning window of the prefill's KV-outer lists (<= 0:
    the default); returns the previous value.  Query workspace sizes after
    setting it."""
    return int(load_library().msa_set_attn_window(int(rows)))


def msa_version() -> str:
    return load_library().msa_version().decode()
