"""Shared-prefix decode attention on the GPU against the float64 oracle.

Groups of requests are forked from one prompt each (the C++ allocator shares
the prompt's blocks by reference), then every member appends its own tokens
(copy-on-write of the shared partial tail, block copies on the device).  The
shared-prefix call must equal dense attention over each request's history
(prompt + its own tokens) within the decode tolerances, and agree with the
plain decode call on the same tables.  A group that claims more shared blocks
than its members really share is flagged.
"""
import numpy as np
import pytest

import workloads as W
from oracle import attention as oatt
from tests.paged_batch import as_f64, torch_from_host

pytestmark = pytest.mark.gpu


def _build(sizes, prompts, appends, Hq, Hkv, D, B, dtype, seed):
    """Fork each group's prompt to its members, append their own tokens; return
    device pools/tables and the per-request host histories."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    g = W.rng(seed)
    S = sum(sizes)
    need = sum(-(-p // B) for p in prompts) + sum(-(-(a + B) // B) + 1 for a in appends) + 8
    N = need
    alloc = pkv.BlockAllocator(N, B, free_order=W.free_order(g, N))
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    kp = torch.full((N, B, Hkv, D), float("nan"), dtype=dt, device="cuda")
    vp = torch.full((N, B, Hkv, D), float("nan"), dtype=dt, device="cuda")
    draw = (lambda shape: W.normal_bf16_bits(g, shape)) if dtype == "bf16" else (lambda shape: W.normal_f32(g, shape))
    member_prompt = [p for p, n in zip(prompts, sizes) for _ in range(n)]
    max_len = max(p + a for p, a in zip(member_prompt, appends))
    maxb = -(-max_len // B) + 1
    group_start = [0]
    hist_k, hist_v = [None] * S, [None] * S
    s0 = 0
    for gi, (n, P) in enumerate(zip(sizes, prompts)):
        assert alloc.add_seq(s0, P) == 0
        pk, pv = draw((P, Hkv, D)), draw((P, Hkv, D))
        if P:
            tab, _ = alloc.fill_tables([s0], maxb)
            slots = pkv.slot_mapping(torch.from_numpy(tab).cuda(), torch.arange(P, dtype=torch.int32, device="cuda"),
                                     B, rows=torch.zeros(P, dtype=torch.int32, device="cuda"))
            pkv.kv_append(torch_from_host(pk), torch_from_host(pv), slots, kp, vp)
        for i in range(1, n):
            assert alloc.fork(s0, s0 + i) == 0
        for i in range(n):
            hist_k[s0 + i], hist_v[s0 + i] = [pk], [pv]
        s0 += n
        group_start.append(s0)
    # every member appends its own tokens, one step at a time
    remaining = list(appends)
    while any(remaining):
        ids = [s for s in range(S) if remaining[s] > 0]
        rc, per, copies = alloc.append(ids)
        assert rc == 0
        if copies:
            pkv.block_copy([kp], [vp], torch.tensor(copies, dtype=torch.int32, device="cuda"))
        tab, lens = alloc.fill_tables(ids, maxb)
        slots = pkv.slot_mapping(torch.from_numpy(tab).cuda(), torch.from_numpy(lens - 1).cuda(), B)
        nk, nv = draw((len(ids), Hkv, D)), draw((len(ids), Hkv, D))
        pkv.kv_append(torch_from_host(nk), torch_from_host(nv), slots, kp, vp)
        for j, s in enumerate(ids):
            hist_k[s].append(nk[j:j + 1])
            hist_v[s].append(nv[j:j + 1])
            remaining[s] -= 1
    assert alloc.check()
    tables, lens = alloc.fill_tables(list(range(S)), maxb)
    hk = [np.concatenate(h) for h in hist_k]
    hv = [np.concatenate(h) for h in hist_v]
    q = draw((S, Hq, D))
    return kp, vp, tables, lens, hk, hv, q, np.array(group_start, np.int32)


@pytest.mark.parametrize("Hq,Hkv,D,B,dtype,sizes", [
    (16, 4, 128, 16, "bf16", (4, 1, 3, 4, 2)),
    (8, 4, 64, 8, "f32", (3, 2, 1, 3)),
    (32, 8, 128, 16, "bf16", (2, 4, 1)),
    (16, 4, 128, 4, "bf16", (4, 2, 3)),    # block size 4: tensor-core tiles laid out block by block
])
def test_shared_prefix_matches_oracle_and_plain_decode(Hq, Hkv, D, B, dtype, sizes):
    import torch

    import paged_kv_cache_358_b200 as pkv

    prompts = [37 * (i + 1) + 5 * i for i in range(len(sizes))]       # 37, 79, 121, ...
    prompts[len(sizes) // 2] = 0                                       # one group with no prompt
    S = sum(sizes)
    appends = [(7 * s) % 23 + (s % 3) * 11 for s in range(S)]          # 0 .. 44 own tokens
    kp, vp, tables, lens, hk, hv, q, gs = _build(sizes, prompts, appends, Hq, Hkv, D, B, dtype, seed=len(sizes))
    # shared full blocks: the prompt's full blocks (a partial tail is copied on the first append)
    pb = np.array([p // B for p in prompts], np.int32)
    for gi in range(len(sizes)):
        members = range(gs[gi], gs[gi + 1])
        for s in members:
            assert (tables[s, :pb[gi]] == tables[gs[gi], :pb[gi]]).all()
    max_group = max(sizes)
    td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    qd = torch_from_host(q)
    scale = 1.0 / np.sqrt(D)
    ws = pkv.shared_prefix_workspace(S, len(sizes), max_group, Hq, Hkv, D, tables.shape[1])
    out = pkv.paged_decode_attn_shared_prefix(qd, kp, vp, td, ld, torch.from_numpy(gs).cuda(),
                                              torch.from_numpy(pb).cuda(), max_group, scale,
                                              out_dtype=torch.float32, workspace=ws)
    assert pkv.decode_status(ws) == 0
    plain = pkv.paged_decode_attn(qd, kp, vp, td, ld, scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    got, ref_plain = as_f64(out), as_f64(plain)
    tol = 1e-2 if dtype == "bf16" else 1e-5
    assert np.all(np.isfinite(got))
    for s in range(S):
        assert hk[s].shape[0] == lens[s]
        ref = oatt.dense_decode(q[s], hk[s], hv[s], scale)
        assert np.max(np.abs(got[s] - ref)) <= tol, f"request {s}"
    assert np.max(np.abs(got - ref_plain)) <= 2 * tol


def test_shared_prefix_flags_a_false_claim():
    import torch

    import paged_kv_cache_358_b200 as pkv

    Hq, Hkv, D, B = 16, 4, 128, 16
    sizes, prompts = (2, 2), (40, 0)
    appends = [3, 5, 20, 9]
    kp, vp, tables, lens, hk, hv, q, gs = _build(sizes, prompts, appends, Hq, Hkv, D, B, "bf16", seed=7)
    # the second group shares nothing, but claims one block
    pb = np.array([40 // B, 1], np.int32)
    ws = pkv.shared_prefix_workspace(4, 2, 2, Hq, Hkv, D, tables.shape[1])
    pkv.paged_decode_attn_shared_prefix(torch_from_host(q), kp, vp, torch.from_numpy(tables).cuda(),
                                        torch.from_numpy(lens).cuda(), torch.from_numpy(gs).cuda(),
                                        torch.from_numpy(pb).cuda(), 2, 1.0 / np.sqrt(D), workspace=ws)
    assert pkv.decode_status(ws) == pkv.Status.BAD_TABLE
    # a fault of an earlier call is not reported again: a valid call on the
    # same workspace (its shared-part status word included) reports OK, and
    # so does a valid call on a workspace full of stale bytes
    pb_ok = np.array([40 // B, 0], np.int32)
    for fill in (None, 0xFF):
        if fill is not None:
            ws.fill_(fill)
        out = pkv.paged_decode_attn_shared_prefix(torch_from_host(q), kp, vp, torch.from_numpy(tables).cuda(),
                                                  torch.from_numpy(lens).cuda(), torch.from_numpy(gs).cuda(),
                                                  torch.from_numpy(pb_ok).cuda(), 2, 1.0 / np.sqrt(D),
                                                  out_dtype=torch.float32, workspace=ws)
        assert pkv.decode_status(ws) == pkv.Status.OK
        got = as_f64(out)
        for s in range(4):
            assert np.max(np.abs(got[s] - oatt.dense_decode(q[s], hk[s], hv[s], 1.0 / np.sqrt(D)))) <= 1e-2


def test_shared_prefix_rejects_unsupported_groups():
    import torch

    import paged_kv_cache_358_b200 as pkv

    L = pkv.lib()
    assert L.pkv_shared_prefix_workspace_bytes(8, 2, 4, 16, 4, 128, 10) > 0
    assert L.pkv_shared_prefix_workspace_bytes(8, 2, 5, 16, 4, 128, 10) == 0     # 5 x 4 columns > 16
    assert L.pkv_shared_prefix_workspace_bytes(8, 2, 17, 8, 8, 128, 10) == 0     # more than 16 members
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.pkv_paged_decode_attn_shared_prefix(z.data_ptr(), z.data_ptr(), z.data_ptr(), z.data_ptr(), 1,
                                               z.data_ptr(), 4, z.data_ptr(), z.data_ptr(), 5, 2, 16, 4, 128,
                                               16, 1, 0.1, pkv.BF16, z.data_ptr(), pkv.BF16, z.data_ptr(), 1 << 20,
                                               None)
    assert rc == pkv.Status.INVALID                                              # more groups than requests


@pytest.mark.parametrize("fill", [0xFF, 0x7F])
def test_shared_prefix_16_columns_with_stale_workspace(fill):
    """16 columns per KV head (4 members x 4 grouped heads): the combine merges
    the shared-part pass's split pieces itself.  Workspace bytes left by
    anything else (NaN or huge values) must not reach an output: CTAs without
    tiles never write their slots, and the merge must not read them.  With 44
    shared tiles over all workers, most workers own none and every split pair
    spans many of them."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    Hq, Hkv, D, B = 16, 4, 128, 16
    sizes, prompts = (4, 3, 4), (150, 40, 0)
    S = sum(sizes)
    appends = [(5 * s) % 17 + 1 for s in range(S)]
    kp, vp, tables, lens, hk, hv, q, gs = _build(sizes, prompts, appends, Hq, Hkv, D, B, "bf16", seed=11)
    pb = np.array([p // B for p in prompts], np.int32)
    ws = pkv.shared_prefix_workspace(S, len(sizes), 4, Hq, Hkv, D, tables.shape[1])
    scale = 1.0 / np.sqrt(D)
    ws.fill_(fill)
    for _ in range(2):   # the second call sees what the first left behind
        out = pkv.paged_decode_attn_shared_prefix(torch_from_host(q), kp, vp, torch.from_numpy(tables).cuda(),
                                                  torch.from_numpy(lens).cuda(), torch.from_numpy(gs).cuda(),
                                                  torch.from_numpy(pb).cuda(), 4, scale,
                                                  out_dtype=torch.float32, workspace=ws)
        assert pkv.decode_status(ws) == pkv.Status.OK
        got = as_f64(out)
        assert np.all(np.isfinite(got))
        for s in range(S):
            assert np.max(np.abs(got[s] - oatt.dense_decode(q[s], hk[s], hv[s], scale))) <= 1e-2, f"request {s}"
