"""Python binding of libsparse_attn.so (the C ABI in include/sparse_attn.h).

Argument marshalling only: torch supplies device memory and the current CUDA
stream; every step of the computation runs in the library's CUDA kernels.
There is no CPU path: inputs must be CUDA tensors and the built library must
be present, otherwise these functions raise.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libsparse_attn.so")

SA_OK = 0
SA_BF16, SA_F32 = 0, 1
STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED", 3: "SA_ERR_CUDA",
                4: "SA_ERR_TIMEOUT", 5: "SA_ERR_DEVICE_ASSERT"}

# Every entry point declared in include/sparse_attn.h and include/sparse_attn_testing.h.
EXPORTED = ("sparse_attn_mask_workspace_bytes", "sparse_attn_mask", "sparse_attn_mask_noalloc",
            "sparse_attn_select", "sparse_attn_bwd_workspace_bytes", "sparse_attn_bwd",
            "sparse_attn_quantize_fp8", "sparse_attn_fwd_fp8",
            "sparse_attn_sparse_linear_workspace_bytes", "sparse_attn_sparse_linear",
            "sparse_attn_kmeans_workspace_bytes", "sparse_attn_kmeans_permutation", "sparse_attn_permute_rows",
            "sparse_attn_fused_workspace_bytes", "sparse_attn_fused",
            "sparse_attn_fwd", "sparse_attn_fwd_dense", "sparse_attn_host_workspace_bytes",
            "sparse_attn_host", "sparse_attn_check_device_error",
            "sparse_attn_last_error", "sparse_attn_version", "sparse_attn_test_fwd_withheld_copy")


class SaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("bq", ctypes.c_int32), ("bk", ctypes.c_int32)]


class SparseAttnError(RuntimeError):
    def __init__(self, func: str, status: int, message: str):
        self.status = status
        super().__init__(f"{func}: {STATUS_NAMES.get(status, status)}: {message}")


_lib = None
_lock = threading.Lock()


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsparse_attn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "block_sparse_attention_row_b200.build.build()")
        lib = ctypes.CDLL(path)
        vp, i32p, u8p, f32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
        sp = ctypes.POINTER(SaShape)
        lib.sparse_attn_mask_workspace_bytes.argtypes = [sp]
        lib.sparse_attn_mask_workspace_bytes.restype = ctypes.c_size_t
        lib.sparse_attn_mask.argtypes = [sp, vp, vp, ctypes.c_double, ctypes.c_double, i32p, i32p,
                                         u8p, f32p, vp, vp]
        lib.sparse_attn_mask.restype = ctypes.c_int
        lib.sparse_attn_mask_noalloc.argtypes = [sp, vp, vp, ctypes.c_double, ctypes.c_double, i32p,
                                                 i32p, u8p, f32p, vp]
        lib.sparse_attn_mask_noalloc.restype = ctypes.c_int
        lib.sparse_attn_select.argtypes = [sp, f32p, ctypes.c_double, ctypes.c_double, i32p, i32p,
                                           u8p, vp]
        lib.sparse_attn_select.restype = ctypes.c_int
        lib.sparse_attn_fwd.argtypes = [sp, vp, vp, vp, i32p, i32p, vp, ctypes.c_int, f32p, vp]
        lib.sparse_attn_fwd.restype = ctypes.c_int
        lib.sparse_attn_fwd_dense.argtypes = [sp, vp, vp, vp, vp, ctypes.c_int, f32p, vp]
        lib.sparse_attn_fwd_dense.restype = ctypes.c_int
        lib.sparse_attn_bwd_workspace_bytes.argtypes = [sp]
        lib.sparse_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.sparse_attn_bwd.argtypes = [sp, vp, vp, vp, vp, vp, f32p, i32p, i32p, vp, vp, vp, ctypes.c_int, vp, vp]
        lib.sparse_attn_bwd.restype = ctypes.c_int
        lib.sparse_attn_quantize_fp8.argtypes = [sp, vp, vp, vp, vp, f32p, f32p, vp]
        lib.sparse_attn_quantize_fp8.restype = ctypes.c_int
        lib.sparse_attn_fwd_fp8.argtypes = [sp, vp, vp, f32p, f32p, vp, i32p, i32p, vp, ctypes.c_int, f32p, vp]
        lib.sparse_attn_fwd_fp8.restype = ctypes.c_int
        lib.sparse_attn_sparse_linear_workspace_bytes.argtypes = [sp]
        lib.sparse_attn_sparse_linear_workspace_bytes.restype = ctypes.c_size_t
        lib.sparse_attn_sparse_linear.argtypes = [sp, vp, vp, vp, i32p, i32p, vp, f32p, vp, ctypes.c_int, vp,
                                                  ctypes.c_size_t, vp]
        lib.sparse_attn_sparse_linear.restype = ctypes.c_int
        lib.sparse_attn_fused_workspace_bytes.argtypes = [sp]
        lib.sparse_attn_fused_workspace_bytes.restype = ctypes.c_size_t
        lib.sparse_attn_fused.argtypes = [sp, vp, vp, vp, ctypes.c_double, ctypes.c_double, i32p, i32p, vp,
                                          ctypes.c_int, f32p, vp, ctypes.c_size_t, vp]
        lib.sparse_attn_fused.restype = ctypes.c_int
        lib.sparse_attn_kmeans_workspace_bytes.argtypes = [sp, ctypes.c_int]
        lib.sparse_attn_kmeans_workspace_bytes.restype = ctypes.c_size_t
        lib.sparse_attn_kmeans_permutation.argtypes = [sp, vp, ctypes.c_int, ctypes.c_int, f32p, i32p, i32p, f32p,
                                                       vp, ctypes.c_size_t, vp]
        lib.sparse_attn_kmeans_permutation.restype = ctypes.c_int
        lib.sparse_attn_permute_rows.argtypes = [sp, vp, i32p, vp, ctypes.c_int, ctypes.c_int, vp]
        lib.sparse_attn_permute_rows.restype = ctypes.c_int
        lib.sparse_attn_host_workspace_bytes.argtypes = [sp, ctypes.c_int, ctypes.c_int]
        lib.sparse_attn_host_workspace_bytes.restype = ctypes.c_size_t
        lib.sparse_attn_host.argtypes = [sp, vp, vp, vp, ctypes.c_double, ctypes.c_double, vp, ctypes.c_int,
                                         i32p, i32p, ctypes.c_int, vp, ctypes.c_size_t, vp]
        lib.sparse_attn_host.restype = ctypes.c_int
        lib.sparse_attn_check_device_error.argtypes = [vp]
        lib.sparse_attn_check_device_error.restype = ctypes.c_int
        lib.sparse_attn_last_error.argtypes = []
        lib.sparse_attn_last_error.restype = ctypes.c_char_p
        lib.sparse_attn_test_fwd_withheld_copy.argtypes = [sp, vp, vp, vp, i32p, i32p, vp, ctypes.c_int,
                                                           ctypes.c_uint64, vp]
        lib.sparse_attn_test_fwd_withheld_copy.restype = ctypes.c_int
        lib.sparse_attn_version.argtypes = []
        lib.sparse_attn_version.restype = ctypes.c_char_p
        _lib = lib
        return lib


def _check(func: str, status: int) -> None:
    if status != SA_OK:
        msg = load_library().sparse_attn_last_error().decode(errors="replace")
        raise SparseAttnError(func, status, msg)


def make_shape(B: int, H: int, N: int, d: int, bq: int, bk: int) -> SaShape:
    return SaShape(int(B), int(H), int(N), int(d), int(bq), int(bk))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(*ts: torch.Tensor) -> None:
    ref = ts[0]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("sparse attention runs on CUDA tensors only (no CPU path)")
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("Q, K, V must be contiguous bf16 tensors of shape [B, H, N, d]")
        if t.shape != ref.shape or t.device != ref.device:
            raise ValueError("Q, K, V must share shape and device")


def num_blocks(N: int, bq: int, bk: int):
    return -(-N // bq), -(-N // bk)


def mask_workspace_bytes(B, H, N, d, bq, bk) -> int:
    shape = make_shape(B, H, N, d, bq, bk)
    return int(load_library().sparse_attn_mask_workspace_bytes(ctypes.byref(shape)))


def _check_out(out: dict, name: str, shape, dtype: torch.dtype, device: torch.device) -> None:
    t = out.get(name)
    if t is None:
        return
    if (not isinstance(t, torch.Tensor) or t.dtype != dtype or tuple(t.shape) != tuple(shape)
            or t.device != device or not t.is_contiguous()):
        raise ValueError(f"out['{name}'] must be a contiguous {dtype} tensor of shape "
                         f"{tuple(shape)} on {device}")


def _check_mask_outputs(out: dict, B: int, H: int, n_q: int, n_k: int, device: torch.device) -> None:
    """Caller-provided outputs of the mask: the kernels write them without bounds checks."""
    _check_out(out, "cnt", (B, H, n_q), torch.int32, device)
    _check_out(out, "idx", (B, H, n_q, n_k), torch.int32, device)
    _check_out(out, "mask", (B, H, n_q, n_k), torch.uint8, device)
    _check_out(out, "P", (B, H, n_q, n_k), torch.float32, device)


def sparse_attn_mask(Q: torch.Tensor, K: torch.Tensor, bq: int, bk: int, k: float, p: float, *,
                     want_mask: bool = False, want_P: bool = False, out: Optional[dict] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Block mask of hybrid Top-k+Top-p selection: {'cnt', 'idx'[, 'mask', 'P']}.

    cnt int32 [B,H,n_q]; idx int32 [B,H,n_q,n_k] (first cnt entries valid,
    ascending); mask uint8 [B,H,n_q,n_k]; P fp32 [B,H,n_q,n_k]. Pass `out`
    (a dict holding those tensors) and `workspace` to avoid allocations.
    """
    _check_qkv(Q, K)
    lib = load_library()
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    dev = Q.device
    shape = make_shape(B, H, N, d, bq, bk)
    res = dict(out) if out is not None else {}
    _check_mask_outputs(res, B, H, n_q, n_k, dev)
    if "cnt" not in res:
        res["cnt"] = torch.empty((B, H, n_q), dtype=torch.int32, device=dev)
    if "idx" not in res:
        res["idx"] = torch.empty((B, H, n_q, n_k), dtype=torch.int32, device=dev)
    if want_mask and "mask" not in res:
        res["mask"] = torch.empty((B, H, n_q, n_k), dtype=torch.uint8, device=dev)
    if want_P and "P" not in res:
        res["P"] = torch.empty((B, H, n_q, n_k), dtype=torch.float32, device=dev)
    nbytes = int(lib.sparse_attn_mask_workspace_bytes(ctypes.byref(shape)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    elif (workspace.device != dev or not workspace.is_contiguous()
          or workspace.numel() * workspace.element_size() < nbytes):
        raise ValueError(f"workspace must be a contiguous tensor of at least {nbytes} bytes on {dev}")
    st = lib.sparse_attn_mask(ctypes.byref(shape), _ptr(Q), _ptr(K), float(k), float(p),
                              _ptr(res["cnt"]), _ptr(res["idx"]), _ptr(res.get("mask")),
                              _ptr(res.get("P")), _ptr(workspace), _stream(dev, stream))
    _check("sparse_attn_mask", st)
    return res


def _header_constant(name: str) -> int:
    """An integer macro of include/sparse_attn.h, read from the header itself."""
    import re
    path = os.path.join(os.path.dirname(PKG_DIR), "include", "sparse_attn.h")
    with open(path) as f:
        m = re.search(r"#define\s+" + name + r"\s+\(([^)]*)\)", f.read())
    if m is None:
        raise RuntimeError(f"{name} is not defined in {path}")
    expr = m.group(1).replace("u", "")
    if not re.fullmatch(r"[0-9 *]+", expr):
        raise RuntimeError(f"{name}: unexpected definition {m.group(1)!r}")
    value = 1
    for factor in expr.split("*"):
        value *= int(factor)
    return value


NOALLOC_SCRATCH_BYTES = _header_constant("SPARSE_ATTN_NOALLOC_SCRATCH_BYTES")


def sparse_attn_mask_noalloc(Q: torch.Tensor, K: torch.Tensor, bq: int, bk: int, k: float,
                             p: float, *, out: dict, stream=None) -> dict:
    """sparse_attn_mask for callers that cannot allocate device memory on the call path.

    The library uses its own fixed 32 MiB device scratch instead of a workspace,
    so this call allocates nothing: the caller passes every output in `out`
    ('cnt', 'idx', and optionally 'mask' and 'P', shaped as for
    sparse_attn_mask). Shapes needing a larger workspace are rejected. Calls
    that run concurrently on the GPU share the scratch and must not overlap.
    """
    _check_qkv(Q, K)
    lib = load_library()
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    if "cnt" not in out or "idx" not in out:
        raise ValueError("out must hold 'cnt' and 'idx' (this entry point allocates nothing)")
    _check_mask_outputs(out, B, H, n_q, n_k, Q.device)
    shape = make_shape(B, H, N, d, bq, bk)
    st = lib.sparse_attn_mask_noalloc(ctypes.byref(shape), _ptr(Q), _ptr(K), float(k), float(p),
                                      _ptr(out["cnt"]), _ptr(out["idx"]), _ptr(out.get("mask")),
                                      _ptr(out.get("P")), _stream(Q.device, stream))
    _check("sparse_attn_mask_noalloc", st)
    return out


def sparse_attn_select(P: torch.Tensor, N: int, d: int, bq: int, bk: int, k: float, p: float, *,
                       want_mask: bool = False, stream=None) -> dict:
    """Selection alone on a given fp32 score matrix P [B,H,n_q,n_k]."""
    if not P.is_cuda or P.dtype != torch.float32 or not P.is_contiguous() or P.dim() != 4:
        raise ValueError("P must be a contiguous fp32 CUDA tensor [B, H, n_q, n_k]")
    lib = load_library()
    B, H, n_q, n_k = P.shape
    if (n_q, n_k) != num_blocks(N, bq, bk):
        raise ValueError("P's block counts do not match N, bq, bk")
    shape = make_shape(B, H, N, d, bq, bk)
    dev = P.device
    res = {"cnt": torch.empty((B, H, n_q), dtype=torch.int32, device=dev),
           "idx": torch.empty((B, H, n_q, n_k), dtype=torch.int32, device=dev)}
    if want_mask:
        res["mask"] = torch.empty((B, H, n_q, n_k), dtype=torch.uint8, device=dev)
    st = lib.sparse_attn_select(ctypes.byref(shape), _ptr(P), float(k), float(p), _ptr(res["cnt"]),
                                _ptr(res["idx"]), _ptr(res.get("mask")), _stream(dev, stream))
    _check("sparse_attn_select", st)
    return res


def _out_tensor(Q: torch.Tensor, out: Optional[torch.Tensor], out_dtype: torch.dtype):
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
    if out is None:
        return torch.empty(Q.shape, dtype=out_dtype, device=Q.device)
    if out.dtype != out_dtype or out.shape != Q.shape or not out.is_contiguous() or out.device != Q.device:
        raise ValueError("out must be a contiguous tensor of Q's shape and out_dtype")
    return out


def sparse_attn_fwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, cnt: torch.Tensor,
                    idx: torch.Tensor, bq: int, bk: int, *, want_lse: bool = False,
                    out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    out_dtype: torch.dtype = torch.bfloat16, stream=None):
    """Block-sparse attention over the kept blocks: O [B,H,N,d] (, lse fp32 [B,H,N]).

    O is bf16 by default; out_dtype=torch.float32 returns the kernel's fp32
    result, of which the bf16 output is the round-to-nearest-even."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    for t, shp in ((cnt, (B, H, n_q)), (idx, (B, H, n_q, n_k))):
        if t.dtype != torch.int32 or not t.is_contiguous() or tuple(t.shape) != shp or t.device != Q.device:
            raise ValueError(f"index tensor must be contiguous int32 {shp} on {Q.device}")
    lib = load_library()
    shape = make_shape(B, H, N, d, bq, bk)
    O = _out_tensor(Q, out, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    st = lib.sparse_attn_fwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(cnt), _ptr(idx),
                             _ptr(O), SA_F32 if O.dtype == torch.float32 else SA_BF16, _ptr(lse),
                             _stream(Q.device, stream))
    _check("sparse_attn_fwd", st)
    return (O, lse) if want_lse else O


def sparse_attn_fwd_dense(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, bq: int, bk: int, *,
                          want_lse: bool = False, out: Optional[torch.Tensor] = None,
                          lse: Optional[torch.Tensor] = None,
                          out_dtype: torch.dtype = torch.bfloat16, stream=None):
    """Same kernel with every key block kept (full attention)."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    lib = load_library()
    shape = make_shape(B, H, N, d, bq, bk)
    O = _out_tensor(Q, out, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    st = lib.sparse_attn_fwd_dense(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                   SA_F32 if O.dtype == torch.float32 else SA_BF16, _ptr(lse),
                                   _stream(Q.device, stream))
    _check("sparse_attn_fwd_dense", st)
    return (O, lse) if want_lse else O


def sparse_attn_quantize_fp8(Q: torch.Tensor, K: torch.Tensor, bq: int, bk: int, *, out: Optional[dict] = None,
                             stream=None) -> dict:
    """Per-block e4m3 codes of Q and K: {'Q8', 'K8' (uint8 [B,H,N,d]), 'q_scale'
    fp32 [B,H,n_q], 'k_scale' fp32 [B,H,n_k]}; x is approximately code * scale."""
    _check_qkv(Q, K)
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    dev = Q.device
    res = dict(out) if out is not None else {}
    for name, shp, dt in (("Q8", Q.shape, torch.uint8), ("K8", Q.shape, torch.uint8),
                          ("q_scale", (B, H, n_q), torch.float32), ("k_scale", (B, H, n_k), torch.float32)):
        if name in res:
            _check_out(res, name, shp, dt, dev)
        else:
            res[name] = torch.empty(shp, dtype=dt, device=dev)
    shape = make_shape(B, H, N, d, bq, bk)
    st = load_library().sparse_attn_quantize_fp8(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(res["Q8"]),
                                                 _ptr(res["K8"]), _ptr(res["q_scale"]), _ptr(res["k_scale"]),
                                                 _stream(dev, stream))
    _check("sparse_attn_quantize_fp8", st)
    return res


def sparse_attn_fwd_fp8(q8: dict, V: torch.Tensor, cnt: torch.Tensor, idx: torch.Tensor, bq: int, bk: int, *,
                        want_lse: bool = False, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16, stream=None):
    """Block-sparse attention with the score product in FP8: q8 is the dict of
    sparse_attn_quantize_fp8; V bf16. Returns O (, lse)."""
    _check_qkv(V)
    B, H, N, d = V.shape
    n_q, n_k = num_blocks(N, bq, bk)
    dev = V.device
    for name, shp, dt in (("Q8", V.shape, torch.uint8), ("K8", V.shape, torch.uint8),
                          ("q_scale", (B, H, n_q), torch.float32), ("k_scale", (B, H, n_k), torch.float32)):
        if name not in q8:
            raise ValueError(f"q8 must hold '{name}'")
        _check_out(q8, name, shp, dt, dev)
    for t, shp in ((cnt, (B, H, n_q)), (idx, (B, H, n_q, n_k))):
        if t.dtype != torch.int32 or not t.is_contiguous() or tuple(t.shape) != shp or t.device != dev:
            raise ValueError(f"index tensor must be contiguous int32 {shp} on {dev}")
    O = _out_tensor(V, out, out_dtype)
    if want_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    shape = make_shape(B, H, N, d, bq, bk)
    st = load_library().sparse_attn_fwd_fp8(ctypes.byref(shape), _ptr(q8["Q8"]), _ptr(q8["K8"]),
                                            _ptr(q8["q_scale"]), _ptr(q8["k_scale"]), _ptr(V), _ptr(cnt),
                                            _ptr(idx), _ptr(O), SA_F32 if O.dtype == torch.float32 else SA_BF16,
                                            _ptr(lse), _stream(dev, stream))
    _check("sparse_attn_fwd_fp8", st)
    return (O, lse) if want_lse else O


def sparse_linear_workspace_bytes(B, H, N, d, bq, bk) -> int:
    shape = make_shape(B, H, N, d, bq, bk)
    return int(load_library().sparse_attn_sparse_linear_workspace_bytes(ctypes.byref(shape)))


def sparse_attn_sparse_linear(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, cnt: torch.Tensor,
                              idx: torch.Tensor, O_s: torch.Tensor, alpha: torch.Tensor, bq: int, bk: int, *,
                              out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                              stream=None) -> torch.Tensor:
    """O = alpha * O_s + (1 - alpha) * O_l: O_s the sparse branch's output
    (sparse_attn_fwd, bf16 or fp32; O takes its dtype), O_l linear attention
    (elu + 1 features) over the complement of each row's kept blocks; alpha
    fp32 [B, H, N]. d = 128."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    dev = Q.device
    for t, shp in ((cnt, (B, H, n_q)), (idx, (B, H, n_q, n_k))):
        if t.dtype != torch.int32 or not t.is_contiguous() or tuple(t.shape) != shp or t.device != dev:
            raise ValueError(f"index tensor must be contiguous int32 {shp} on {dev}")
    if O_s.dtype not in (torch.bfloat16, torch.float32) or O_s.shape != Q.shape or not O_s.is_contiguous() \
            or O_s.device != dev:
        raise ValueError("O_s must be a contiguous bf16 or fp32 tensor of Q's shape")
    if alpha.dtype != torch.float32 or tuple(alpha.shape) != (B, H, N) or not alpha.is_contiguous() \
            or alpha.device != dev:
        raise ValueError(f"alpha must be a contiguous fp32 tensor {(B, H, N)} on {dev}")
    O = _out_tensor(Q, out, O_s.dtype)
    lib = load_library()
    shape = make_shape(B, H, N, d, bq, bk)
    nbytes = int(lib.sparse_attn_sparse_linear_workspace_bytes(ctypes.byref(shape)))
    if nbytes == 0:
        raise ValueError("unsupported shape for the sparse + linear path (d must be 128)")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    wbytes = workspace.numel() * workspace.element_size()
    st = lib.sparse_attn_sparse_linear(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(cnt), _ptr(idx),
                                       _ptr(O_s), _ptr(alpha), _ptr(O),
                                       SA_F32 if O.dtype == torch.float32 else SA_BF16, _ptr(workspace), wbytes,
                                       _stream(dev, stream))
    _check("sparse_attn_sparse_linear", st)
    return O


def fused_workspace_bytes(B, H, N, d, bq, bk) -> int:
    shape = make_shape(B, H, N, d, bq, bk)
    return int(load_library().sparse_attn_fused_workspace_bytes(ctypes.byref(shape)))


def sparse_attn_fused(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, bq: int, bk: int, k: float, p: float, *,
                      out_dtype=torch.bfloat16, want_lse: bool = False, out: Optional[dict] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Mask and attention in one cooperative kernel launch (SpargeAttention2
    §2C). Returns {"O", "cnt", "idx"} (and "lse"), bit-equal to
    sparse_attn_mask followed by sparse_attn_fwd."""
    _check_qkv(Q, K, V)
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    dev = Q.device
    out = {} if out is None else out
    for key, shp, dt in (("cnt", (B, H, n_q), torch.int32), ("idx", (B, H, n_q, n_k), torch.int32),
                         ("lse", (B, H, N), torch.float32)):
        if key == "lse" and not want_lse:
            continue
        if key not in out:
            out[key] = torch.empty(shp, dtype=dt, device=dev)
        t = out[key]
        if t.dtype != dt or tuple(t.shape) != shp or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"out[{key!r}] must be a contiguous {dt} tensor {shp} on {dev}")
    out["O"] = _out_tensor(Q, out.get("O"), out_dtype)
    lib = load_library()
    shape = make_shape(B, H, N, d, bq, bk)
    nbytes = int(lib.sparse_attn_fused_workspace_bytes(ctypes.byref(shape)))
    if nbytes == 0:
        raise ValueError("unsupported shape for the single-launch path (n_k above its shared-memory limit?)")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    st = lib.sparse_attn_fused(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), float(k), float(p), _ptr(out["cnt"]),
                               _ptr(out["idx"]), _ptr(out["O"]), SA_F32 if out_dtype == torch.float32 else SA_BF16,
                               _ptr(out.get("lse")), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(dev, stream))
    _check("sparse_attn_fused", st)
    return out


def kmeans_workspace_bytes(B, H, N, d, C, bq: int = 64, bk: int = 64) -> int:
    shape = make_shape(B, H, N, d, bq, bk)
    return int(load_library().sparse_attn_kmeans_workspace_bytes(ctypes.byref(shape), int(C)))


def sparse_attn_kmeans_permutation(X: torch.Tensor, C: int, iters: int, *, init: Optional[torch.Tensor] = None,
                                   out_centroids: Optional[torch.Tensor] = None,
                                   workspace: Optional[torch.Tensor] = None, stream=None):
    """k-means of every head's token vectors (Sparse VideoGen2 §2A) and the
    stable permutation by cluster. X bf16 [B, H, N, d]; init fp32
    [B, H, C, d] (cached centroids) or None; out_centroids: where the final
    centroids go (may be init itself: the cache updated in place). Returns
    (ids int32 [B, H, N], perm int32 [B, H, N], centroids fp32 [B, H, C, d])."""
    if not isinstance(X, torch.Tensor) or not X.is_cuda or X.dtype != torch.bfloat16 or X.dim() != 4 \
            or not X.is_contiguous():
        raise ValueError("X must be a contiguous bf16 CUDA tensor [B, H, N, d]")
    B, H, N, d = X.shape
    dev = X.device
    if init is not None and (init.dtype != torch.float32 or tuple(init.shape) != (B, H, int(C), d)
                             or not init.is_contiguous() or init.device != dev):
        raise ValueError(f"init must be a contiguous fp32 tensor {(B, H, int(C), d)} on {dev}")
    lib = load_library()
    shape = make_shape(B, H, N, d, 64, 64)
    nbytes = int(lib.sparse_attn_kmeans_workspace_bytes(ctypes.byref(shape), int(C)))
    if nbytes == 0:
        raise ValueError(f"unsupported shape or C={C} for the k-means permutation")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ids = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    perm = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    if out_centroids is None:
        M = torch.empty((B, H, int(C), d), dtype=torch.float32, device=dev)
    else:
        M = out_centroids
        if M.dtype != torch.float32 or tuple(M.shape) != (B, H, int(C), d) or not M.is_contiguous() or M.device != dev:
            raise ValueError(f"out_centroids must be a contiguous fp32 tensor {(B, H, int(C), d)} on {dev}")
    st = lib.sparse_attn_kmeans_permutation(ctypes.byref(shape), _ptr(X), int(C), int(iters), _ptr(init),
                                            _ptr(ids), _ptr(perm), _ptr(M), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(), _stream(dev, stream))
    _check("sparse_attn_kmeans_permutation", st)
    return ids, perm, M


def sparse_attn_permute_rows(X: torch.Tensor, perm: torch.Tensor, *, inverse: bool = False,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y[b, h, i] = X[b, h, perm[b, h, i]] (inverse: Y[b, h, perm[b, h, i]] =
    X[b, h, i]). X bf16 or fp32 [B, H, N, d]; perm int32 [B, H, N]."""
    if not isinstance(X, torch.Tensor) or not X.is_cuda or X.dtype not in (torch.bfloat16, torch.float32) \
            or X.dim() != 4 or not X.is_contiguous():
        raise ValueError("X must be a contiguous bf16 or fp32 CUDA tensor [B, H, N, d]")
    B, H, N, d = X.shape
    dev = X.device
    if perm.dtype != torch.int32 or tuple(perm.shape) != (B, H, N) or not perm.is_contiguous() \
            or perm.device != dev:
        raise ValueError(f"perm must be a contiguous int32 tensor {(B, H, N)} on {dev}")
    Y = _out_tensor(X, out, X.dtype)
    if Y.data_ptr() == X.data_ptr():
        raise ValueError("out must not be X")
    shape = make_shape(B, H, N, d, 64, 64)
    st = load_library().sparse_attn_permute_rows(ctypes.byref(shape), _ptr(X), _ptr(perm), _ptr(Y),
                                                 SA_F32 if X.dtype == torch.float32 else SA_BF16,
                                                 1 if inverse else 0, _stream(dev, stream))
    _check("sparse_attn_permute_rows", st)
    return Y


def bwd_workspace_bytes(B, H, N, d, bq, bk) -> int:
    shape = make_shape(B, H, N, d, bq, bk)
    return int(load_library().sparse_attn_bwd_workspace_bytes(ctypes.byref(shape)))


def sparse_attn_bwd(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, O: torch.Tensor, dO: torch.Tensor,
                    lse: torch.Tensor, cnt: torch.Tensor, idx: torch.Tensor, bq: int, bk: int, *,
                    out_dtype: torch.dtype = torch.float32, out: Optional[dict] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None):
    """Gradients (dQ, dK, dV) of sparse_attn_fwd for the upstream gradient dO,
    with the kept-block lists held fixed. O and lse are the forward's bf16
    output and log-sum-exp. Outputs are fp32 (default) or bf16."""
    _check_qkv(Q, K, V, O, dO)
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    dev = Q.device
    for t, shp, dt in ((cnt, (B, H, n_q), torch.int32), (idx, (B, H, n_q, n_k), torch.int32),
                       (lse, (B, H, N), torch.float32)):
        if t.dtype != dt or not t.is_contiguous() or tuple(t.shape) != shp or t.device != dev:
            raise ValueError(f"cnt, idx, lse must be contiguous {dt} {shp} on {dev}")
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
    res = dict(out) if out is not None else {}
    for name in ("dQ", "dK", "dV"):
        if name in res:
            _check_out(res, name, Q.shape, out_dtype, dev)
        else:
            res[name] = torch.empty(Q.shape, dtype=out_dtype, device=dev)
    lib = load_library()
    shape = make_shape(B, H, N, d, bq, bk)
    nbytes = int(lib.sparse_attn_bwd_workspace_bytes(ctypes.byref(shape)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    elif (workspace.device != dev or not workspace.is_contiguous()
          or workspace.numel() * workspace.element_size() < nbytes):
        raise ValueError(f"workspace must be a contiguous tensor of at least {nbytes} bytes on {dev}")
    st = lib.sparse_attn_bwd(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse),
                             _ptr(cnt), _ptr(idx), _ptr(res["dQ"]), _ptr(res["dK"]), _ptr(res["dV"]),
                             SA_F32 if out_dtype == torch.float32 else SA_BF16, _ptr(workspace),
                             _stream(dev, stream))
    _check("sparse_attn_bwd", st)
    return res["dQ"], res["dK"], res["dV"]


def sparse_attn(Q, K, V, bq: int, bk: int, k: float, p: float, *, stream=None):
    """The whole path: mask then block-sparse forward. Returns (O, cnt, idx)."""
    m = sparse_attn_mask(Q, K, bq, bk, k, p, stream=stream)
    O = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], bq, bk, stream=stream)
    return O, m["cnt"], m["idx"]


def permuted_sparse_attn(Q, K, V, bq: int, bk: int, k: float, p: float, C_q: int, C_k: int, iters: int, *,
                         init_q: Optional[torch.Tensor] = None, init_k: Optional[torch.Tensor] = None,
                         stream=None) -> dict:
    """Sparse VideoGen2 §2A ahead of the path: Q and K clustered independently
    (k-means, C_q and C_k clusters, `iters` rounds, optional cached centroids),
    Q rows and K, V rows gathered into cluster order, the mask and block-sparse
    forward run on the permuted sequences, and O scattered back to token order.
    Returns {"O", "cnt", "idx" (of the permuted sequence), "perm_q", "perm_k",
    "centroids_q", "centroids_k"}."""
    _, perm_q, Mq = sparse_attn_kmeans_permutation(Q, C_q, iters, init=init_q, stream=stream)
    _, perm_k, Mk = sparse_attn_kmeans_permutation(K, C_k, iters, init=init_k, stream=stream)
    Qp = sparse_attn_permute_rows(Q, perm_q, stream=stream)
    Kp = sparse_attn_permute_rows(K, perm_k, stream=stream)
    Vp = sparse_attn_permute_rows(V, perm_k, stream=stream)
    Op, cnt, idx = sparse_attn(Qp, Kp, Vp, bq, bk, k, p, stream=stream)
    O = sparse_attn_permute_rows(Op, perm_q, inverse=True, stream=stream)
    return {"O": O, "cnt": cnt, "idx": idx, "perm_q": perm_q, "perm_k": perm_k,
            "centroids_q": Mq, "centroids_k": Mk}


def host_workspace_bytes(B: int, H: int, N: int, d: int, bq: int, bk: int,
                         out_dtype=torch.bfloat16, heads_per_chunk: int = 0) -> int:
    od = SA_F32 if out_dtype == torch.float32 else SA_BF16
    sh = make_shape(B, H, N, d, bq, bk)
    n = load_library().sparse_attn_host_workspace_bytes(ctypes.byref(sh), od, int(heads_per_chunk))
    if n == 0:
        raise ValueError("unsupported shape, output type or heads_per_chunk")
    return int(n)


def sparse_attn_host(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, bq: int, bk: int, k: float, p: float,
                     *, device=None, out_dtype=torch.bfloat16, want_cnt: bool = False, want_idx: bool = False,
                     heads_per_chunk: int = 0, out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None,
                     stream=None) -> dict:
    """The whole path on host tensors (page-locked for overlap): copies, mask and
    attention pipelined by chunks of heads on the library's streams.

    Returns host tensors {"O", and "cnt"/"idx" if requested}; they are ready
    once `stream` (default: the device's current stream) has reached this call.
    """
    for t in (Q, K, V):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("Q, K, V must be contiguous bf16 host tensors of shape [B, H, N, d]")
        if t.shape != Q.shape:
            raise ValueError("Q, K, V must share shape")
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if dev.type != "cuda":
        raise ValueError("device must be a CUDA device")
    B, H, N, d = Q.shape
    n_q, n_k = num_blocks(N, bq, bk)
    od = SA_F32 if out_dtype == torch.float32 else SA_BF16
    pin = Q.is_pinned()
    out = {} if out is None else out
    if "O" not in out:
        out["O"] = torch.empty(B, H, N, d, dtype=out_dtype, pin_memory=pin)
    if want_cnt and "cnt" not in out:
        out["cnt"] = torch.empty(B, H, n_q, dtype=torch.int32, pin_memory=pin)
    if want_idx and "idx" not in out:
        out["idx"] = torch.empty(B, H, n_q, n_k, dtype=torch.int32, pin_memory=pin)
    need = host_workspace_bytes(B, H, N, d, bq, bk, out_dtype, heads_per_chunk)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    sh = make_shape(B, H, N, d, bq, bk)
    st = load_library().sparse_attn_host(
        ctypes.byref(sh), _ptr(Q), _ptr(K), _ptr(V), float(k), float(p), _ptr(out["O"]), od,
        _ptr(out.get("cnt") if want_cnt else None), _ptr(out.get("idx") if want_idx else None),
        int(heads_per_chunk), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(dev, stream))
    _check("sparse_attn_host", st)
    out["workspace"] = workspace
    return out


def check_device_error(device=None, stream=None) -> None:
    """Synchronise and raise if a kernel recorded an error since the last check."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    st = load_library().sparse_attn_check_device_error(_stream(dev, stream))
    _check("sparse_attn_check_device_error", st)


def version() -> str:
    return load_library().sparse_attn_version().decode()
