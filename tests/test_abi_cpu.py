"""The C-ABI library builds, loads and exports every symbol include/msa.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(msa_[a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    return msa.load_library()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for want in ("msa_index_topk", "msa_sparse_attn_prefill", "msa_sparse_attn_decode", "msa_combine"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    from block_sparse_long_exp_b200 import msa
    names = _declared_functions()
    assert sorted(set(msa.EXPORTED)) == names
    for n in names:
        assert hasattr(lib, n), n


def test_version_string(lib):
    from block_sparse_long_exp_b200 import msa
    assert "sm_100a" in msa.msa_version()


def test_host_validation_without_gpu(lib):
    from block_sparse_long_exp_b200 import msa
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = (ctypes.c_int32 * 2)(0, 1024)
    seqs = msa.Varlen(1, 1024, 1024, 0, 1024, 1024, ctypes.addressof(cu), ctypes.addressof(cu))
    # supported shapes get a workspace size; unsupported ones get 0
    assert lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(seqs)) >= 256
    assert lib.msa_sparse_attn_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), 0) > 1024 * 4 * 16 * 16 * 128 * 2
    bad = msa.make_shape(64, 4, 96, 64, 16)           # d = 96 is not built
    assert lib.msa_index_topk_workspace_size(ctypes.byref(bad), ctypes.byref(seqs)) == 0
    bad_bk = msa.make_shape(64, 4, 128, 64, 16, B_k=96)            # block sizes: 32, 64, 128
    assert lib.msa_sparse_attn_workspace_size(ctypes.byref(bad_bk), ctypes.byref(seqs), 0) == 0
    for bk in (32, 64):
        sh = msa.make_shape(64, 4, 128, 64, 16, B_k=bk)
        assert lib.msa_sparse_attn_workspace_size(ctypes.byref(sh), ctypes.byref(seqs), 0) > 0
        assert lib.msa_index_topk_workspace_size(ctypes.byref(sh), ctypes.byref(seqs)) >= 256
    # entry points reject invalid arguments before any launch
    rc = lib.msa_index_topk(ctypes.byref(shape), ctypes.byref(seqs), None, None, None, None, 0, None)
    assert rc == 1                                       # MSA_ERR_INVALID_ARG
    rc = lib.msa_index_topk(ctypes.byref(bad), ctypes.byref(seqs), 1, 1, 1, 1, 1 << 20, None)
    assert rc == 2                                       # MSA_ERR_UNSUPPORTED
    rc = lib.msa_index_topk(None, ctypes.byref(seqs), 1, 1, 1, 1, 1 << 20, None)
    assert rc == 1
    rc = lib.msa_sparse_attn_prefill(ctypes.byref(shape), ctypes.byref(seqs), 256, 256, 256, 256, 256, None,
                                     0, 256, 16, None)
    assert rc == 3                                       # MSA_ERR_WORKSPACE (16 bytes is too small)
    not_gqa = msa.make_shape(64, 3, 128, 64, 16)
    rc = lib.msa_combine(ctypes.byref(not_gqa), 4, 1, 1, 1, 1, None, None)
    assert rc == 1                                       # H % G != 0
    more_q_than_k = msa.Varlen(1, 2048, 1024, 0, 2048, 1024, ctypes.addressof(cu), ctypes.addressof(cu))
    rc = lib.msa_index_topk(ctypes.byref(shape), ctypes.byref(more_q_than_k), 1, 1, 1, 1, 1 << 20, None)
    assert rc == 1


def test_paged_decode_host_validation_without_gpu(lib):
    from block_sparse_long_exp_b200 import msa
    shape = msa.make_shape(64, 4, 128, 64, 16)
    lens = (ctypes.c_int32 * 2)(1000, 300)
    table = (ctypes.c_int32 * 16)(*range(16))
    ok = msa.Paged(2, 8, 1000, 0, 64, ctypes.addressof(lens), ctypes.addressof(table))
    assert lib.msa_decode_paged_workspace_size(ctypes.byref(shape), ctypes.byref(ok)) >= 256
    # lengths beyond the table, missing pointers, too many pages: rejected before any launch
    too_long = msa.Paged(2, 8, 8 * 128 + 1, 0, 64, ctypes.addressof(lens), ctypes.addressof(table))
    assert lib.msa_decode_paged_workspace_size(ctypes.byref(shape), ctypes.byref(too_long)) == 0
    no_table = msa.Paged(2, 8, 1000, 0, 64, ctypes.addressof(lens), None)
    rc = lib.msa_index_topk_decode_paged(ctypes.byref(shape), ctypes.byref(no_table), 1, 1, 1, 1, 1 << 20, None)
    assert rc == 1                                       # MSA_ERR_INVALID_ARG
    huge = msa.Paged(2, 8, 1000, 0, 1 << 26, ctypes.addressof(lens), ctypes.addressof(table))
    rc = lib.msa_sparse_attn_decode_paged(ctypes.byref(shape), ctypes.byref(huge), 1, 1, 1, 1, 1, None, 1, 1 << 20,
                                          None)
    assert rc == 2                                       # MSA_ERR_UNSUPPORTED (rows past int32)
    rc = lib.msa_sparse_attn_decode_paged(ctypes.byref(shape), ctypes.byref(ok), 1, 1, 1, 1, 1, None, 256, 16, None)
    assert rc == 3                                       # MSA_ERR_WORKSPACE


def test_tile_threshold_setting_round_trips(lib):
    from block_sparse_long_exp_b200 import msa
    prev = msa.msa_set_tile_threshold(0)
    try:
        assert msa.msa_set_tile_threshold(7) == 0
        assert msa.msa_set_tile_threshold(-5) == 7        # any negative value means automatic
        assert msa.msa_set_tile_threshold(-1) == -1
    finally:
        msa.msa_set_tile_threshold(prev)


def test_plain_c_program_uses_the_boundary(lib, tmp_path):
    """A C program that includes only include/msa.h and links libmsa.so."""
    import shutil
    import subprocess
    from block_sparse_long_exp_b200 import msa
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(msa.LIB_PATH)
    exe = tmp_path / "abi_host"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", libdir, "-lmsa",
                    "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "abi_host ok" in r.stdout


def test_limits_and_empty_calls_answer_before_any_launch(lib):
    """Prefill-shaped index calls take at most 1024 sequences: the workspace query
    returns 0 and the call MSA_ERR_UNSUPPORTED before anything is launched.
    A call with no queries still obeys the workspace rule."""
    from block_sparse_long_exp_b200 import msa
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = (ctypes.c_int32 * 2)(0, 0)
    many = msa.Varlen(1025, 2, 2, 0, 2050, 2050, ctypes.addressof(cu), ctypes.addressof(cu))
    assert lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(many)) == 0
    rc = lib.msa_index_topk(ctypes.byref(shape), ctypes.byref(many), 256, 256, 256, 256, 1 << 20, None)
    assert rc == 2                                       # MSA_ERR_UNSUPPORTED
    decode_shaped = msa.Varlen(1025, 1, 2, 0, 1025, 2050, ctypes.addressof(cu), ctypes.addressof(cu))
    assert lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(decode_shaped)) > 0
    empty = msa.Varlen(1, 0, 10, 0, 0, 10, ctypes.addressof(cu), ctypes.addressof(cu))
    for fn in (lib.msa_sparse_attn_prefill,):
        rc = fn(ctypes.byref(shape), ctypes.byref(empty), None, None, None, None, None, None, 0, None, 0, None)
        assert rc == 3                                   # MSA_ERR_WORKSPACE: no workspace given
    rc = lib.msa_dense_attn(ctypes.byref(shape), ctypes.byref(empty), None, None, None, None, None, None, 0, None)
    assert rc == 3
    rc = lib.msa_index_topk(ctypes.byref(shape), ctypes.byref(empty), None, None, None, None, 0, None)
    assert rc == 3


def test_lengths_beyond_their_totals_are_rejected(lib):
    from block_sparse_long_exp_b200 import msa
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = (ctypes.c_int32 * 2)(0, 0)
    for bad in (msa.Varlen(1, 300, 400, 0, 200, 400, ctypes.addressof(cu), ctypes.addressof(cu)),    # max_q > total_q
                msa.Varlen(1, 100, 500, 0, 100, 400, ctypes.addressof(cu), ctypes.addressof(cu))):   # max_k > total_k
        assert lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(bad)) == 0
        rc = lib.msa_index_topk(ctypes.byref(shape), ctypes.byref(bad), 256, 256, 256, 256, 1 << 20, None)
        assert rc == 1                                   # MSA_ERR_INVALID_ARG


def test_index_kl_host_validation_without_gpu(lib):
    from block_sparse_long_exp_b200 import msa
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = (ctypes.c_int32 * 2)(0, 0)
    seqs = msa.Varlen(1, 300, 300, 0, 300, 300, ctypes.addressof(cu), ctypes.addressof(cu))
    args = (256, 256, 256, 256)
    rc = lib.msa_index_kl(ctypes.byref(shape), ctypes.byref(seqs), *args, None, 256, 0.5, 0, 256, None, 256, 1 << 20,
                          None)
    assert rc == 1                                       # sparse support without a selection
    rc = lib.msa_index_kl(ctypes.byref(shape), ctypes.byref(seqs), *args, 256, 256, float("nan"), 0, 256, None, 256,
                          1 << 20, None)
    assert rc == 1                                       # tau must be finite
    rc = lib.msa_index_kl(ctypes.byref(shape), ctypes.byref(seqs), *args, None, 256, 0.5, 1, 256, None, 256, 16, None)
    assert rc == 3                                       # dense: no selection needed, but the workspace is
    bad = msa.make_shape(64, 4, 96, 64, 16)
    rc = lib.msa_index_kl(ctypes.byref(bad), ctypes.byref(seqs), *args, 256, 256, 0.5, 0, 256, None, 256, 1 << 20,
                          None)
    assert rc == 2                                       # d = 96 is not built
    rc = lib.msa_index_kl_backward(ctypes.byref(shape), ctypes.byref(seqs), *args, 256, 256, None, 0.5, 0, 256, 256,
                                   256, 1 << 20, None)
    assert rc == 1                                       # the backward needs the student's log-sum-exp


def test_training_workspaces_and_backward_checks_without_gpu(lib):
    # the selected support's KL target, KL gradient and Main Branch backward
    # plan the forward's KV-outer lists in their workspace; the dense support
    # takes the 256-byte header alone
    from block_sparse_long_exp_b200 import msa
    H, G, d, d_idx, k = 64, 4, 128, 64, 16
    shape = msa.make_shape(H, G, d, d_idx, k)
    T = 1024
    cu = (ctypes.c_int32 * 2)(0, T)
    seqs = msa.Varlen(1, T, T, 0, T, T, ctypes.addressof(cu), ctypes.addressof(cu))
    sz_kl = lib.msa_index_kl_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), 0)
    sz_bwd = lib.msa_sparse_attn_backward_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), 0)
    assert lib.msa_index_kl_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), 1) == 256
    assert lib.msa_sparse_attn_backward_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), 1) == 256
    entries = T * G * k * 4                              # one packed entry per (query, group, slot)
    assert sz_kl >= 256 + entries + T * G * k * 16       # the target's float4 partial per slot
    assert sz_bwd >= 256 + entries + T * H * 4           # the backward's D per (query, head)
    # the same plan, then their own tails (each rounded to the workspace alignment)
    assert abs((sz_kl - sz_bwd) - (T * G * k * 16 - T * H * 4)) <= 512
    bad = msa.make_shape(H, G, 96, d_idx, k)             # d = 96 is not built
    assert lib.msa_sparse_attn_backward_workspace_size(ctypes.byref(bad), ctypes.byref(seqs), 0) == 0
    # the selected support reads q / out / dout and adds dq rows 16 bytes at a time
    args = dict(q=256, k=256, v=256, sel=256, out=256, lse=256, dout=256, dq=256, dk=256, dv=256)

    def bwd(ws_bytes, dense=0, **over):
        a = {**args, **over}
        return lib.msa_sparse_attn_backward(ctypes.byref(shape), ctypes.byref(seqs), a["q"], a["k"], a["v"], a["sel"],
                                            a["out"], a["lse"], a["dout"], dense, a["dq"], a["dk"], a["dv"], 256,
                                            ws_bytes, None)
    for name in ("q", "out", "dout", "dq"):
        assert bwd(sz_bwd, **{name: 264}) == 1, name
    assert bwd(sz_bwd - 256) == 3                        # one plan's worth of workspace is required
    assert bwd(sz_bwd, k=264) == 1                       # key rows on every support


def test_selected_share_host_checks(lib):
    assert lib.msa_selected_share(None, None, 0, None, None) == 0       # nothing to do
    assert lib.msa_selected_share(None, 256, 5, 256, None) == 1
    assert lib.msa_selected_share(256, 256, -1, 256, None) == 1


def test_gather_pages_host_checks(lib):
    from block_sparse_long_exp_b200 import msa
    cu = (ctypes.c_int32 * 2)(0, 0)
    table = (ctypes.c_int32 * 8)(*range(8))
    seqs = msa.Varlen(1, 900, 900, 0, 900, 900, ctypes.addressof(cu), ctypes.addressof(cu))
    T = ctypes.addressof(table)
    assert lib.msa_gather_pages(ctypes.byref(seqs), None, 8, 8, 128, 256, 256, 256, 1 << 20, None) == 1  # no table
    assert lib.msa_gather_pages(ctypes.byref(seqs), T, 7, 8, 128, 256, 256, 256, 1 << 20, None) == 1     # 900 > 7 * 128
    assert lib.msa_gather_pages(ctypes.byref(seqs), T, 8, 8, 100, 256, 256, 256, 1 << 20, None) == 1     # row bytes
    assert lib.msa_gather_pages(ctypes.byref(seqs), T, 8, 8, 128, 258, 256, 256, 1 << 20, None) == 1     # alignment
    assert lib.msa_gather_pages(ctypes.byref(seqs), T, 8, 8, 128, 256, 256, 256, 16, None) == 3          # workspace


def test_noalloc_host_checks_match_msa_index_topk(lib):
    """The allocation-free decode index call checks its arguments as
    msa_index_topk does, in the same order, before it looks anything up on a
    device: a bad shape or sequence description gives the same status, and the
    data pointers are only required when there are queries."""
    from block_sparse_long_exp_b200 import msa
    shape = msa.make_shape(64, 4, 128, 64, 16)
    bad_bk = msa.make_shape(64, 4, 128, 64, 16, B_k=96)
    cu = (ctypes.c_int32 * 3)(0, 1, 2)
    cuk = (ctypes.c_int32 * 3)(0, 500, 900)
    seqs = msa.Varlen(2, 1, 500, 0, 2, 900, ctypes.addressof(cu), ctypes.addressof(cuk))
    no_cu = msa.Varlen(2, 1, 500, 0, 2, 900, None, ctypes.addressof(cuk))

    def both(sh, sq, ptr):
        a = lib.msa_index_topk(sh, sq, ptr, ptr, ptr, None, 0, None)
        b = lib.msa_index_topk_decode_noalloc(sh, sq, ptr, ptr, ptr, None, None)
        return a, b

    a, b = both(ctypes.byref(shape), ctypes.byref(no_cu), 256)
    assert a == b == 1                                   # MSA_ERR_INVALID_ARG: null cu_q
    a, b = both(ctypes.byref(bad_bk), ctypes.byref(seqs), 256)
    assert a == b == 2                                   # MSA_ERR_UNSUPPORTED: B_k = 96
    a, b = both(None, ctypes.byref(seqs), 256)
    assert a == b == 1
    # queries present: null data pointers are rejected
    assert lib.msa_index_topk_decode_noalloc(ctypes.byref(shape), ctypes.byref(seqs), None, None, None, None,
                                             None) == 1
    # no queries: null data pointers are allowed (without a GPU the call then
    # stops at the device lookup, never at the argument check)
    none_q = msa.Varlen(2, 0, 500, 0, 0, 900, ctypes.addressof(cu), ctypes.addressof(cuk))
    rc = lib.msa_index_topk_decode_noalloc(ctypes.byref(shape), ctypes.byref(none_q), None, None, None, None, None)
    assert rc != 1


def test_selftest_wait_host_checks(lib):
    """The bounded-wait self-test rejects a limit outside 1 us ... 1 s and a
    missing or short workspace before it launches anything."""
    n = lib.msa_selftest_wait_timeout_workspace_size()
    assert n >= 264
    assert lib.msa_selftest_wait_timeout(0, 256, n, None) == 1            # MSA_ERR_INVALID_ARG
    assert lib.msa_selftest_wait_timeout(1000001, 256, n, None) == 1
    assert lib.msa_selftest_wait_timeout(1000, None, n, None) == 3        # MSA_ERR_WORKSPACE
    assert lib.msa_selftest_wait_timeout(1000, 256, n - 1, None) == 3
    assert lib.msa_selftest_wait_timeout(1000, 272, n, None) == 3         # not 256-byte aligned


def test_block_size_128_only_entry_points(lib):
    """B_k = 32 / 64 run on the main path (index top-k, sparse attention,
    decode); the training-side kernels, the selection variants and paged
    caches are built for 128-token blocks and say so before any launch."""
    from block_sparse_long_exp_b200 import msa
    sh64 = msa.make_shape(64, 4, 128, 64, 16, B_k=64)
    cu = (ctypes.c_int32 * 2)(0, 1024)
    seqs = msa.Varlen(1, 1024, 1024, 0, 1024, 1024, ctypes.addressof(cu), ctypes.addressof(cu))
    U = 2                                                # MSA_ERR_UNSUPPORTED
    assert lib.msa_select_window(ctypes.byref(sh64), ctypes.byref(seqs), 1, 256, 256, 1 << 20, None) == U
    assert lib.msa_index_topk_policy(ctypes.byref(sh64), ctypes.byref(seqs), 1, 1, 256, 256, 256, 256, 1 << 20,
                                     None) == U
    lens = (ctypes.c_int32 * 1)(1000)
    table = (ctypes.c_int32 * 8)(*range(8))
    pages = msa.Paged(1, 8, 1000, 0, 8, ctypes.addressof(lens), ctypes.addressof(table))
    assert lib.msa_decode_paged_workspace_size(ctypes.byref(sh64), ctypes.byref(pages)) == 0


def test_fused_prefill_host_checks(lib):
    """msa_prefill answers bad arguments before any launch: decode shapes and
    more than 1024 sequences are refused, NULL data pointers with queries are
    invalid, a short workspace is refused; its workspace is the main branch's
    for the same pass size; the overlap setter returns the previous value."""
    from block_sparse_long_exp_b200 import msa
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = (ctypes.c_int32 * 2)(0, 0)
    a = ctypes.addressof(cu)
    seqs = msa.Varlen(1, 4096, 4096, 0, 4096, 4096, a, a)
    for q_chunk in (0, 1024, 700):
        need = lib.msa_prefill_workspace_size(ctypes.byref(shape), ctypes.byref(seqs), q_chunk)
        assert need > 0 and need == lib.msa_sparse_attn_workspace_size(ctypes.byref(shape), ctypes.byref(seqs),
                                                                       q_chunk)
    decode = msa.Varlen(4, 1, 4096, 0, 4, 16384, a, a)
    assert lib.msa_prefill_workspace_size(ctypes.byref(shape), ctypes.byref(decode), 0) == 0
    p = [256] * 8
    rc = lib.msa_prefill(ctypes.byref(shape), ctypes.byref(decode), *p, 0, 256, 1 << 30, None)
    assert rc == 1                                       # MSA_ERR_INVALID_ARG: decode shapes have their own calls
    many = msa.Varlen(1025, 2, 2, 0, 2050, 2050, a, a)
    assert lib.msa_prefill_workspace_size(ctypes.byref(shape), ctypes.byref(many), 0) == 0
    rc = lib.msa_prefill(ctypes.byref(shape), ctypes.byref(many), *p, 0, 256, 1 << 30, None)
    assert rc == 2                                       # MSA_ERR_UNSUPPORTED
    for i in range(7):                                   # q k v q_idx k_idx sel out (lse may be NULL)
        q = list(p)
        q[i] = None
        rc = lib.msa_prefill(ctypes.byref(shape), ctypes.byref(seqs), *q, 0, 256, 1 << 30, None)
        assert rc == 1, i
    rc = lib.msa_prefill(ctypes.byref(shape), ctypes.byref(seqs), *p, 0, 256, 16, None)
    assert rc == 3                                       # MSA_ERR_WORKSPACE
    bad_bk = msa.make_shape(64, 4, 128, 64, 16, B_k=96)
    rc = lib.msa_prefill(ctypes.byref(bad_bk), ctypes.byref(seqs), *p, 0, 256, 1 << 30, None)
    assert rc == 2
    rc = lib.msa_prefill(None, ctypes.byref(seqs), *p, 0, 256, 1 << 30, None)
    assert rc == 1
    prev = lib.msa_set_prefill_overlap(16)
    try:
        assert lib.msa_set_prefill_overlap(0) == 16
        assert lib.msa_set_prefill_overlap(-5) == 0      # < 0: back to the default
        assert lib.msa_set_prefill_overlap(prev) == 0    # the default: no overlap
    finally:
        lib.msa_set_prefill_overlap(prev)
