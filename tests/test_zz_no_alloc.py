"""The allocation-free decode entry point against the workspace one.

pkv_paged_decode_attn_noalloc exists for callers that cannot allocate device
memory themselves (a plugin whose host runtime owns every device allocation,
a serving loop that must never call cudaMalloc).  It keeps its scratch in an
array built into the library, shared by every call on a device.  This test
calls it through the C ABI on three different batches in a row (one with 16
grouped heads per KV head, whose split pieces a second launch merges), and
checks each result against pkv_paged_decode_attn with a caller workspace and
against the float64 oracle, so a second call that picked up state left by the
first would fail.  It also checks that a batch whose stated workspace size is
beyond the built-in scratch is refused, for both storage types.

This file is collected last so that a run stopping at the first failure has
already run every other test; it passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from tests.paged_batch import as_f64, device_batch, host_batch, oracle_out

pytestmark = pytest.mark.gpu


def _noalloc(db, wl, out):
    import torch

    import paged_kv_cache_358_b200 as pkv

    rc = pkv.lib().pkv_paged_decode_attn_noalloc(
        db.q.data_ptr(), db.k_pool.data_ptr(), db.v_pool.data_ptr(), db.tables.data_ptr(), db.max_blocks,
        db.seq_lens.data_ptr(), db.q.shape[0], wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
        wl.pool_blocks, ctypes.c_float(wl.scale), pkv.BF16 if wl.dtype == "bf16" else pkv.F32,
        out.data_ptr(), pkv.F32, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


def test_noalloc_matches_workspace_entry_point_on_successive_calls():
    import torch

    import paged_kv_cache_358_b200 as pkv

    # 16 grouped heads per KV head: the 16-column tiles, whose split pieces
    # the second launch merges from the same built-in scratch
    lens16 = tuple(list(W.workload("mixed_512").lengths)[:200])
    wl16 = W.DecodeWorkload("g16", 1, 32, 2, 128, 16, "bf16", lens16,
                            pool_blocks=sum(-(-n // 16) for n in lens16) + 8, seed=5)
    cases = [(W.workload("mixed_512", block_size=16), list(W.workload("mixed_512").lengths)[:300], 1e-2),
             (W.workload("tiny"), None, 1e-5),
             (wl16, None, 1e-2)]
    for wl, lengths, tol in cases:
        hb = host_batch(wl, lengths=lengths)
        db = device_batch(hb)
        got = torch.full(db.q.shape, float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(db, wl, got) == pkv.Status.OK
        ref = pkv.paged_decode_attn(db.q, db.k_pool, db.v_pool, db.tables, db.seq_lens, wl.scale,
                                    out_dtype=torch.float32)
        torch.cuda.synchronize()
        g, r = as_f64(got), as_f64(ref)
        assert np.all(np.isfinite(g))
        assert np.max(np.abs(g - r)) <= tol
        assert np.max(np.abs(g - oracle_out(hb))) <= tol


@pytest.mark.parametrize("kv_dtype", ["bf16", "f32"])
def test_noalloc_refuses_batches_beyond_its_scratch(kv_dtype):
    import torch

    import paged_kv_cache_358_b200 as pkv

    Hq, Hkv, D = 32, 8, 128
    # the smallest batch whose stated workspace size exceeds 16 MiB is refused,
    # the largest one within it runs
    lo, hi = 1, 1 << 16
    while lo < hi:
        mid = (lo + hi) // 2
        if pkv.decode_workspace_bytes(mid, Hq, Hkv, D) > (16 << 20):
            hi = mid
        else:
            lo = mid + 1
    S_over = lo
    assert pkv.decode_workspace_bytes(S_over - 1, Hq, Hkv, D) <= (16 << 20)
    dt = torch.bfloat16 if kv_dtype == "bf16" else torch.float32
    code = pkv.BF16 if kv_dtype == "bf16" else pkv.F32
    q = torch.zeros((S_over, Hq, D), dtype=dt, device="cuda")
    pool = torch.zeros((4, 16, Hkv, D), dtype=dt, device="cuda")
    t = torch.zeros((S_over, 1), dtype=torch.int32, device="cuda")
    lens = torch.zeros((S_over,), dtype=torch.int32, device="cuda")
    out = torch.full((S_over, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    rc = pkv.lib().pkv_paged_decode_attn_noalloc(
        q.data_ptr(), pool.data_ptr(), pool.data_ptr(), t.data_ptr(), 1, lens.data_ptr(), S_over, Hq, Hkv, D, 16,
        4, ctypes.c_float(0.1), code, out.data_ptr(), pkv.F32, None)
    assert rc == pkv.Status.INVALID
    assert "16 MiB" in pkv.lib().pkv_last_cuda_error().decode()
    # one request fewer fits: every length is 0, so every output is 0
    rc = pkv.lib().pkv_paged_decode_attn_noalloc(
        q.data_ptr(), pool.data_ptr(), pool.data_ptr(), t.data_ptr(), 1, lens.data_ptr(), S_over - 1, Hq, Hkv, D,
        16, 4, ctypes.c_float(0.1), code, out.data_ptr(), pkv.F32, None)
    assert rc == pkv.Status.OK
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[:S_over - 1]).item() == 0
