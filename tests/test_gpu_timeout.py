"""Failure detection of the attention kernel: a bounded wait that runs out
(needs a B200).

The test hook sparse_attn_test_fwd_withheld_copy runs the forward with every
pipeline wait bounded by a short limit and withholds one K copy in the first
CTA, so the waits that depend on it cannot complete. Nothing faults or hangs:
the kernel records SA_ERR_TIMEOUT, that CTA drains what it had issued and
returns. The host reads the status, and the next normal call on the same
device must match the oracle.
"""
import ctypes
import re

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (SparseAttnError, capi, check_device_error,
                                             sparse_attn_fwd, sparse_attn_mask)

from _gpu_cases import MAX_ABS_TOL, MEAN_ABS_TOL, all_rows, compare_outputs, custom

# The kernel's wait sites (the info field of the device error record).
WAIT_SITES = {0xE001: "ch_empty", 0xE002: "q_full", 0xE003: "ch_full", 0xE004: "p_full",
              0xE005: "s_full", 0xE006: "o_full", 0xE007: "q_empty", 0xE008: "issue lock",
              0xE009: "staging tile"}


@pytest.mark.gpu
@pytest.mark.parametrize("d,bq", [(128, 128), (64, 64)])
def test_withheld_copy_times_out_then_next_call_is_correct(d, bq):
    B, H, N = 1, 2, 2048
    (Q, K, V), (Qh, Kh, Vh) = custom(B, H, N, d, seed=5 + d, positional_field=True)
    m = sparse_attn_mask(Q, K, bq, 64, 0.3, 0.0)
    lib = capi.load_library()
    shape = capi.make_shape(B, H, N, d, bq, 64)
    O_bad = torch.empty((B, H, N, d), dtype=torch.float32, device=Q.device)
    st = lib.sparse_attn_test_fwd_withheld_copy(
        ctypes.byref(shape), capi._ptr(Q), capi._ptr(K), capi._ptr(V), capi._ptr(m["cnt"]),
        capi._ptr(m["idx"]), capi._ptr(O_bad), capi.SA_F32, 100_000_000,   # 100 ms per wait
        capi._stream(Q.device))
    assert st == capi.SA_OK, lib.sparse_attn_last_error()
    with pytest.raises(SparseAttnError, match="SA_ERR_TIMEOUT") as info:
        check_device_error(Q.device)
    site = int(re.search(r"info 0x([0-9a-f]+)", str(info.value)).group(1), 16)
    print(f"\n[withheld copy d={d} bq={bq}] timed out at {WAIT_SITES.get(site, hex(site))}")
    assert site in WAIT_SITES
    check_device_error(Q.device)   # the record was cleared

    # The device and the library are usable: a normal call matches the oracle.
    O_gpu = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], bq, 64, out_dtype=torch.float32)
    check_device_error(Q.device)
    rows = all_rows(B, H, -(-N // bq))
    O_ref, _ = O.block_sparse_attention(Qh, Kh, Vh, m["cnt"].cpu().numpy(), m["idx"].cpu().numpy(),
                                        bq, 64, rows=rows)
    mx, mean = compare_outputs(O_gpu, O_ref, rows, bq, N)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)


def test_withheld_copy_hook_validates_its_limit():
    """Host side, nothing enqueued: limits outside [1 ms, 4 s] are refused."""
    from block_sparse_attention_row_b200 import build
    build.build()
    lib = capi.load_library()
    shape = capi.make_shape(1, 2, 2048, 128, 128, 64)
    a = ctypes.c_void_p(256)
    for lim in (0, 999_999, 4_000_000_001):
        st = lib.sparse_attn_test_fwd_withheld_copy(ctypes.byref(shape), a, a, a, a, a, a, 0, lim, None)
        assert st == 1, lim
        assert b"wait_limit_ns" in lib.sparse_attn_last_error()
