"""The C-ABI library on the host (no GPU): it builds, loads, exports every
declared entry point, and rejects bad arguments before touching a device."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("sparse_attn.h", "sparse_attn_testing.h")]


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_row_b200 import build
    build.build()
    from block_sparse_attention_row_b200 import capi
    return capi.load_library()


def declared_functions():
    names = set()
    for h in HEADERS:
        names |= set(re.findall(r"\b(sparse_attn_\w+)\s*\(", open(h).read()))
    return sorted(names)


def test_header_declares_the_binding_list():
    from block_sparse_attention_row_b200.capi import EXPORTED
    assert declared_functions() == sorted(EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version(lib):
    assert b"sm_100a" in lib.sparse_attn_version()


@pytest.mark.parametrize("B,H,N,d,bq,bk", [(1, 2, 4096, 64, 64, 64), (1, 40, 32760, 128, 128, 64),
                                           (1, 40, 75600, 128, 128, 64), (2, 24, 17550, 128, 128, 64),
                                           (1, 1, 1, 64, 64, 64)])
def test_workspace_bytes(lib, B, H, N, d, bq, bk):
    from block_sparse_attention_row_b200.capi import make_shape
    n_q, n_k = math.ceil(N / bq), math.ceil(N / bk)
    ld = (n_k + 3) // 4 * 4
    r = lambda x: (x + 255) // 256 * 256
    want = r(B * H * n_q * d * 4) + r(B * H * n_k * d * 4) + r(B * H * n_q * ld * 4)
    sh = make_shape(B, H, N, d, bq, bk)
    assert lib.sparse_attn_mask_workspace_bytes(ctypes.byref(sh)) == want


def test_workspace_bytes_rejects_bad_shapes(lib):
    from block_sparse_attention_row_b200.capi import make_shape
    for args in [(1, 1, 0, 64, 64, 64), (1, 1, 100, 96, 64, 64), (1, 1, 100, 64, 32, 64),
                 (1, 1, 100, 64, 64, 128), (1, 1, 64 * 8193, 64, 64, 64), (300, 300, 64, 64, 64, 64)]:
        sh = make_shape(*args)
        assert lib.sparse_attn_mask_workspace_bytes(ctypes.byref(sh)) == 0, args
    assert lib.sparse_attn_mask_workspace_bytes(None) == 0


def _mask_status(lib, shape, k=0.1, p=0.9, ptr=16):
    p_ = ctypes.c_void_p(ptr)
    return lib.sparse_attn_mask(shape, p_, p_, k, p, p_, p_, None, None, ctypes.c_void_p(256), None)


def test_host_validation_codes(lib):
    from block_sparse_attention_row_b200.capi import make_shape
    good = ctypes.byref(make_shape(1, 2, 4096, 64, 64, 64))
    assert _mask_status(lib, None) == 1
    assert _mask_status(lib, ctypes.byref(make_shape(1, 2, 4096, 96, 64, 64))) == 2
    assert _mask_status(lib, ctypes.byref(make_shape(1, 2, 4096, 64, 64, 32))) == 2
    assert _mask_status(lib, good, k=0.0, p=0.0) == 1
    assert _mask_status(lib, good, k=-0.1) == 1
    assert _mask_status(lib, good, p=1.5) == 1
    assert _mask_status(lib, good, k=float("nan")) == 1
    assert _mask_status(lib, good, ptr=0) == 1           # NULL pointers
    assert _mask_status(lib, good, ptr=8) == 1           # misaligned
    assert b"aligned" in lib.sparse_attn_last_error()
    z = ctypes.c_void_p(0)
    assert lib.sparse_attn_fwd(good, z, z, z, z, z, z, 0, None, None) == 1
    assert lib.sparse_attn_fwd_dense(good, z, z, z, z, 0, None, None) == 1
    a = ctypes.c_void_p(16)
    assert lib.sparse_attn_fwd(good, a, a, a, a, a, a, 7, None, None) == 1   # unknown o_dtype
    assert b"o_dtype" in lib.sparse_attn_last_error()
    assert lib.sparse_attn_select(good, z, 0.1, 0.9, z, z, None, None) == 1
    assert lib.sparse_attn_select(good, ctypes.c_void_p(16), 0.0, 0.0, ctypes.c_void_p(16),
                                  ctypes.c_void_p(16), None, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    from block_sparse_attention_row_b200 import sparse_attn_mask
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        sparse_attn_mask(q, q, 64, 64, 0.1, 0.9)


def test_host_pipeline_workspace_and_validation(lib):
    """sparse_attn_host: chunk planning and host-side argument checks (nothing enqueued)."""
    from block_sparse_attention_row_b200.capi import host_workspace_bytes, make_shape
    r = lambda x: (x + 255) // 256 * 256
    B, H, N, d = 1, 40, 32760, 128
    n_q, n_k = -(-N // 128), -(-N // 64)
    for hpc, out_dtype, esize in ((0, 0, 2), (3, 0, 2), (7, 1, 4), (40, 0, 2), (100, 0, 2)):
        got = lib.sparse_attn_host_workspace_bytes(ctypes.byref(make_shape(B, H, N, d, 128, 64)), out_dtype, hpc)
        h = min(H, -(-2368 // n_q)) if hpc == 0 else min(hpc, H)
        ld = (n_k + 3) // 4 * 4
        mws = r(h * n_q * d * 4) + r(h * n_k * d * 4) + r(h * n_q * ld * 4)
        per = 3 * r(h * N * d * 2) + r(h * N * d * esize) + r(h * n_q * 4) + r(h * n_q * n_k * 4) + r(mws)
        assert got == 2 * per, (hpc, got, 2 * per)
    good = ctypes.byref(make_shape(1, 2, 4096, 64, 64, 64))
    assert lib.sparse_attn_host_workspace_bytes(good, 0, -1) == 0
    assert lib.sparse_attn_host_workspace_bytes(good, 9, 0) == 0
    a = ctypes.c_void_p(16)
    z = ctypes.c_void_p(0)
    need = lib.sparse_attn_host_workspace_bytes(good, 0, 0)
    ws = ctypes.c_void_p(256)
    assert lib.sparse_attn_host(good, a, a, a, 0.1, 0.9, a, 0, None, None, 0, ws, need - 1, None) == 1
    assert b"workspace" in _host_msg(lib)
    assert lib.sparse_attn_host(good, z, a, a, 0.1, 0.9, a, 0, None, None, 0, ws, need, None) == 1
    assert lib.sparse_attn_host(good, a, a, a, 0.0, 0.0, a, 0, None, None, 0, ws, need, None) == 1
    assert lib.sparse_attn_host(good, a, a, a, 0.1, 0.9, a, 0, None, None, 0, ctypes.c_void_p(16), need, None) == 1
    assert lib.sparse_attn_host(good, a, a, a, 0.1, 0.9, a, 5, None, None, 0, ws, need, None) == 1
    assert lib.sparse_attn_host(good, a, a, a, 0.1, 0.9, a, 0, None, None, -2, ws, need, None) == 1
    assert _host_msg(lib).startswith(b"heads_per_chunk")


def _host_msg(lib):
    return lib.sparse_attn_last_error()


def test_mask_output_validation_rejects_wrong_tensors():
    """The caller-provided outputs of the mask are checked before any launch
    (the kernels write them without bounds checks)."""
    import torch
    from block_sparse_attention_row_b200 import capi
    dev = torch.device("cpu")
    good = {"cnt": torch.empty(1, 2, 8, dtype=torch.int32), "idx": torch.empty(1, 2, 8, 16, dtype=torch.int32),
            "mask": torch.empty(1, 2, 8, 16, dtype=torch.uint8), "P": torch.empty(1, 2, 8, 16)}
    capi._check_mask_outputs(good, 1, 2, 8, 16, dev)
    bad = [("cnt", torch.empty(1, 2, 9, dtype=torch.int32)),            # wrong shape
           ("idx", torch.empty(1, 2, 8, 16, dtype=torch.int64)),        # wrong dtype
           ("mask", torch.empty(1, 2, 16, 8, dtype=torch.uint8).transpose(-1, -2)),  # not contiguous
           ("P", torch.empty(1, 2, 8, 15))]
    for name, t in bad:
        with pytest.raises(ValueError, match=name):
            capi._check_mask_outputs({**good, name: t}, 1, 2, 8, 16, dev)
    with pytest.raises(ValueError, match="on cuda"):
        capi._check_mask_outputs(good, 1, 2, 8, 16, torch.device("cuda", 0))


def test_noalloc_scratch_size_is_read_from_the_header():
    from block_sparse_attention_row_b200 import capi
    src = open(HEADERS[0]).read()
    assert "#define SPARSE_ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)" in src
    assert capi.NOALLOC_SCRATCH_BYTES == 32 * 1024 * 1024


@pytest.mark.parametrize("B,H,N,d,bq", [(1, 2, 4096, 64, 64), (1, 40, 32760, 128, 128), (2, 24, 17550, 128, 128),
                                        (1, 3, 777, 64, 64), (1, 1, 1, 128, 128)])
def test_bwd_workspace_bytes(lib, B, H, N, d, bq):
    from block_sparse_attention_row_b200.capi import make_shape
    n_q, n_k = -(-N // bq), -(-N // 64)
    nw, n_kp = -(-n_k // 32), -(-n_k // 2)
    r = lambda x: (x + 255) // 256 * 256
    want = r(B * H * n_q * bq * 8) + r(B * H * n_q * nw * 4) + r(B * H * n_kp * 4) + r(B * H * n_kp * n_q * 4)
    assert lib.sparse_attn_bwd_workspace_bytes(ctypes.byref(make_shape(B, H, N, d, bq, 64))) == want
    assert lib.sparse_attn_bwd_workspace_bytes(ctypes.byref(make_shape(B, H, N, 96, bq, 64))) == 0


def test_bwd_host_validation(lib):
    from block_sparse_attention_row_b200.capi import make_shape
    good = ctypes.byref(make_shape(1, 2, 4096, 64, 64, 64))
    a, z, ws = ctypes.c_void_p(16), ctypes.c_void_p(0), ctypes.c_void_p(256)
    args = [a] * 11
    for pos in range(11):
        bad = list(args)
        bad[pos] = z
        assert lib.sparse_attn_bwd(good, *bad, 1, ws, None) == 1, pos
    assert lib.sparse_attn_bwd(good, *args, 5, ws, None) == 1          # unknown g_dtype
    assert lib.sparse_attn_bwd(good, *args, 1, ctypes.c_void_p(16), None) == 1   # workspace alignment
    bad = list(args)
    bad[3] = ctypes.c_void_p(24)
    assert lib.sparse_attn_bwd(good, *bad, 1, ws, None) == 1
    assert b"aligned" in lib.sparse_attn_last_error()


def test_fp8_host_validation(lib):
    from block_sparse_attention_row_b200.capi import make_shape
    a, z = ctypes.c_void_p(16), ctypes.c_void_p(0)
    d64 = ctypes.byref(make_shape(1, 2, 4096, 64, 64, 64))
    d128 = ctypes.byref(make_shape(1, 2, 4096, 128, 128, 64))
    assert lib.sparse_attn_fwd_fp8(d64, a, a, a, a, a, a, a, a, 0, None, None) == 2    # d = 64 unsupported
    assert b"FP8" in lib.sparse_attn_last_error()
    assert lib.sparse_attn_fwd_fp8(d128, a, a, z, a, a, a, a, a, 0, None, None) == 1   # no q_scale
    assert lib.sparse_attn_fwd_fp8(d128, a, a, a, a, a, a, a, a, 3, None, None) == 1   # o_dtype
    assert lib.sparse_attn_quantize_fp8(d128, a, a, a, z, a, a, None) == 1
    assert lib.sparse_attn_quantize_fp8(d128, a, a, a, ctypes.c_void_p(20), a, a, None) == 1


def test_sparse_linear_host_validation(lib):
    from block_sparse_attention_row_b200.capi import make_shape
    a, z, ws = ctypes.c_void_p(16), ctypes.c_void_p(0), ctypes.c_void_p(256)
    d128 = ctypes.byref(make_shape(1, 2, 4096, 128, 128, 64))
    d64 = ctypes.byref(make_shape(1, 2, 4096, 64, 64, 64))
    need = lib.sparse_attn_sparse_linear_workspace_bytes(d128)
    assert need > 0 and lib.sparse_attn_sparse_linear_workspace_bytes(d64) == 0
    assert lib.sparse_attn_sparse_linear(d64, a, a, a, a, a, a, a, a, 0, ws, need, None) == 2
    assert lib.sparse_attn_sparse_linear(d128, a, a, a, a, a, z, a, a, 0, ws, need, None) == 1
    assert lib.sparse_attn_sparse_linear(d128, a, a, a, a, a, a, a, a, 0, ws, need - 1, None) == 1
    assert b"workspace" in lib.sparse_attn_last_error()
    assert lib.sparse_attn_sparse_linear(d128, a, a, a, a, a, a, a, a, 0, ctypes.c_void_p(16), need, None) == 1


def test_kmeans_host_validation(lib):
    from block_sparse_attention_row_b200.capi import make_shape
    a, z, ws = ctypes.c_void_p(16), ctypes.c_void_p(0), ctypes.c_void_p(256)
    sh = ctypes.byref(make_shape(1, 2, 1000, 128, 64, 64))
    need = lib.sparse_attn_kmeans_workspace_bytes(sh, 100)
    assert need == ((2 * 101 * 4 + 255) // 256) * 256
    for C in (0, -1, 1001):
        assert lib.sparse_attn_kmeans_workspace_bytes(sh, C) == 0
    assert lib.sparse_attn_kmeans_workspace_bytes(ctypes.byref(make_shape(1, 2, 1000, 96, 64, 64)), 10) == 0
    assert lib.sparse_attn_kmeans_permutation(sh, a, 1001, 5, None, a, a, a, ws, need, None) == 1
    assert lib.sparse_attn_kmeans_permutation(sh, a, 100, 101, None, a, a, a, ws, need, None) == 1
    assert lib.sparse_attn_kmeans_permutation(sh, a, 100, -1, None, a, a, a, ws, need, None) == 1
    assert lib.sparse_attn_kmeans_permutation(sh, z, 100, 5, None, a, a, a, ws, need, None) == 1
    assert lib.sparse_attn_kmeans_permutation(sh, a, 100, 5, None, a, a, a, ws, need - 1, None) == 1
    assert b"workspace" in lib.sparse_attn_last_error()
    assert lib.sparse_attn_kmeans_permutation(sh, a, 100, 5, None, a, a, a, ctypes.c_void_p(16), need, None) == 1
    assert lib.sparse_attn_kmeans_permutation(sh, a, 100, 5, ctypes.c_void_p(8), a, a, a, ws, need, None) == 1
    # Row permutation: dtype, aliasing, null and alignment are refused before any launch.
    assert lib.sparse_attn_permute_rows(sh, a, a, ctypes.c_void_p(32), 2, 0, None) == 1
    assert lib.sparse_attn_permute_rows(sh, a, a, a, 0, 0, None) == 1
    assert lib.sparse_attn_permute_rows(sh, a, z, ctypes.c_void_p(32), 0, 0, None) == 1
    assert lib.sparse_attn_permute_rows(sh, a, a, ctypes.c_void_p(40), 0, 0, None) == 1


def test_kmeans_binding_refuses_cpu_tensors():
    import torch
    from block_sparse_attention_row_b200 import sparse_attn_kmeans_permutation, sparse_attn_permute_rows
    X = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sparse_attn_kmeans_permutation(X, 4, 2)
    with pytest.raises(ValueError):
        sparse_attn_permute_rows(X, torch.zeros(1, 1, 64, dtype=torch.int32))


def test_fused_host_validation(lib):
    from block_sparse_attention_row_b200.capi import make_shape
    a, z, ws = ctypes.c_void_p(16), ctypes.c_void_p(0), ctypes.c_void_p(256)
    sh = ctypes.byref(make_shape(1, 2, 4096, 128, 128, 64))
    need = lib.sparse_attn_fused_workspace_bytes(sh)
    n_q, n_k = 32, 64
    assert need == ((2 * n_q * 128 * 4 + 255) // 256) * 256 + ((2 * n_k * 128 * 4 + 255) // 256) * 256 + 256
    # Rows longer than the selection phase's shared memory allows are refused:
    # n_k <= 1549 for d = 128, n_k <= 1344 for d = 64.
    for d, n_max in ((128, 1549), (64, 1344)):
        assert lib.sparse_attn_fused_workspace_bytes(ctypes.byref(make_shape(1, 1, 64 * n_max, d, 128, 64))) > 0
        assert lib.sparse_attn_fused_workspace_bytes(ctypes.byref(make_shape(1, 1, 64 * n_max + 1, d, 128, 64))) == 0
    big = ctypes.byref(make_shape(1, 1, 64 * 1550, 128, 128, 64))
    assert lib.sparse_attn_fused(big, a, a, a, 0.05, 0.9, a, a, a, 0, None, ws, 1 << 30, None) == 2
    assert lib.sparse_attn_fused(sh, a, a, a, 0.0, 0.0, a, a, a, 0, None, ws, need, None) == 1   # k = p = 0
    assert lib.sparse_attn_fused(sh, z, a, a, 0.05, 0.9, a, a, a, 0, None, ws, need, None) == 1
    assert lib.sparse_attn_fused(sh, a, a, a, 0.05, 0.9, a, a, a, 3, None, ws, need, None) == 1
    assert lib.sparse_attn_fused(sh, a, a, a, 0.05, 0.9, a, a, a, 0, None, ws, need - 1, None) == 1
    assert lib.sparse_attn_fused(sh, a, a, a, 0.05, 0.9, a, a, a, 0, None, ctypes.c_void_p(16), need, None) == 1
    assert lib.sparse_attn_fused(sh, a, a, a, 0.05, 0.9, a, a, a, 0, None, z, need, None) == 1
