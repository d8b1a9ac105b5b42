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


def test_topk_count_matches_oracle_rule():
    import oracle
    from block_sparse_attention_row_b200 import topk_count
    for k in (0.0, 0.03, 0.05, 0.07, 0.1, 0.125, 0.25, 0.5, 0.999, 1.0):
        for n in (1, 7, 64, 100, 256, 275, 512, 1182):
            assert topk_count(k, n) == oracle.topk_count(k, n)


def test_exp2_poly_constants_come_from_the_remez_script():
    """The kernel's polynomial constants are the ones the derivation script prints."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "gen_exp2_poly", os.path.join(ROOT, "block_sparse_attention_row_b200", "csrc", "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    coef, err = gen.remez_relative()
    assert err < 1e-4
    src = open(os.path.join(ROOT, "block_sparse_attention_row_b200", "csrc", "sa_attn_kernel.cuh")).read()
    body = src[src.index("float exp2_poly("):src.index("return (x == -INFINITY)")]
    lits = [float(v) for v in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]
    assert len(lits) == 4
    c3, c2, c1, c0 = lits
    import numpy as np
    assert np.allclose([c0, c1, c2, c3], np.float32(coef), rtol=0, atol=2e-9)


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
