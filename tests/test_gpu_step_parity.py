"""The decode step exactly as the benchmark times it, at its full size, against
the float64 oracle.

Workload: 32 requests with a 4096-token history, H_q 32, H_kv 8, d 128, bf16,
block size 16, shuffled free queue.  Each step runs what a caller runs per
decode iteration: the C++ allocator reserves one slot per request, the tables
and lengths are mirrored to the device, the slot mapping and the plan run
once, then every layer makes one launch that appends the new token's K/V and
attends ([P2] "PagedAttention：让 KV cache 按需生长", sections "写满一块，再拿下一块"
and "分页以后，attention 仍然按完整历史归一化").  Layers after the first are
launched with programmatic dependent launch (pkv_set_launch_overlap), whose
early loads read the pools and tables before the previous launch completes;
the result must not depend on that timing.

Two consecutive steps over 4 layers: step 2 attends over the row step 1
appended.  Checked:
* per layer and step, 48 sampled (request, query head) outputs against dense
  attention over the history plus the appended rows (bf16 output: 1e-2 plus
  half a bf16 ulp of the value);
* outputs and pools bit-identical with launch overlap off;
* the appended rows are in the pools bit for bit; the device status word is 0.
"""
import numpy as np
import pytest

import workloads as W
from oracle import attention as oatt
from tests.paged_batch import as_f64, bf16_out_tol, device_batch, host_batch, torch_from_host

pytestmark = pytest.mark.gpu

LAYERS = 4
STEPS = 2
SAMPLES = 48


def _run(pkv, torch, hb, db, base_pools, qs, kn, vn, overlap):
    """Run STEPS decode steps over LAYERS layers from the same starting state;
    return per step the outputs of every layer, the slots, and the pools."""
    wl = hb.wl
    S, Hq, Hkv, D, B = len(hb.lengths), wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
    alloc = pkv.BlockAllocator(wl.pool_blocks, B, free_order=hb.order)
    ids = np.arange(S, dtype=np.int32)
    for i, n in enumerate(hb.lengths):
        assert alloc.add_seq(i, n) == 0
    pools = [(k.clone(), v.clone()) for k, v in base_pools]
    ws = pkv.new_workspace(S, Hq, Hkv, D)
    status = np.zeros(S, dtype=np.int32)
    copies = np.zeros((S, 3), dtype=np.int32)
    steps = []
    for step in range(STEPS):
        rc, nc = alloc.append_arrays(ids, status, copies)
        assert rc == 0 and nc == 0
        tables, lens = alloc.fill_tables(ids, db.max_blocks)
        td = torch.from_numpy(tables).cuda()
        ld = torch.from_numpy(lens).cuda()
        slots = pkv.slot_mapping(td, torch.from_numpy(lens - 1).cuda(), B)
        pkv.decode_plan(ld, Hq, Hkv, D, pkv.BF16, ws)
        outs = []
        try:
            for layer in range(LAYERS):
                out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device="cuda")
                # the first layer follows the plan kernel, which writes what it reads first
                pkv.set_launch_overlap(overlap and layer > 0)
                kp, vp = pools[layer]
                pkv.paged_decode_attn_append_run(qs[step][layer], kn[step][layer], vn[step][layer], slots, kp, vp,
                                                 td, ld, wl.scale, out, ws)
                outs.append(out)
        finally:
            pkv.set_launch_overlap(False)
        torch.cuda.synchronize()
        assert pkv.decode_status(ws) == 0
        steps.append((outs, slots.clone(), lens.copy()))
    assert alloc.check()
    return steps, pools


def test_benchmarked_step_full_size_matches_oracle():
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl = W.workload("teaching_32x4096", decode_steps=STEPS + 2)
    hb = host_batch(wl)
    S, Hq, Hkv, D, B = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
    G = Hq // Hkv
    max_blocks = -(-(max(hb.lengths) + STEPS) // B) + 1
    db = device_batch(hb, max_blocks=max_blocks)
    # per-layer pools with distinct contents: layer l holds the history rolled
    # by l along head_dim (an input transform applied identically on both sides)
    base = [(torch.roll(db.k_pool, l, dims=3).contiguous(), torch.roll(db.v_pool, l, dims=3).contiguous())
            for l in range(LAYERS)]
    del db.k_pool, db.v_pool
    g = W.rng(4242)
    qs_h = [[W.normal_bf16_bits(g, (S, Hq, D)) for _ in range(LAYERS)] for _ in range(STEPS)]
    kn_h = [[W.normal_bf16_bits(g, (S, Hkv, D)) for _ in range(LAYERS)] for _ in range(STEPS)]
    vn_h = [[W.normal_bf16_bits(g, (S, Hkv, D)) for _ in range(LAYERS)] for _ in range(STEPS)]
    qs = [[torch_from_host(x) for x in row] for row in qs_h]
    kn = [[torch_from_host(x) for x in row] for row in kn_h]
    vn = [[torch_from_host(x) for x in row] for row in vn_h]

    plain, pools_plain = _run(pkv, torch, hb, db, base, qs, kn, vn, overlap=False)
    over, pools_over = _run(pkv, torch, hb, db, base, qs, kn, vn, overlap=True)

    # launch overlap changes nothing
    for (oa, sa, _), (ob, sb, _) in zip(plain, over):
        assert torch.equal(sa, sb)
        for x, y in zip(oa, ob):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    for (ka, va), (kb, vb) in zip(pools_plain, pools_over):
        assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
        assert torch.equal(va.view(torch.int16), vb.view(torch.int16))

    # appended rows landed in their slots
    for step, (_, slots, _) in enumerate(over):
        sl = slots.cpu().numpy()
        for layer in range(LAYERS):
            kp, vp = pools_over[layer]
            kflat = kp.view(-1, Hkv, D).view(torch.int16)
            vflat = vp.view(-1, Hkv, D).view(torch.int16)
            got_k = kflat[torch.from_numpy(sl).cuda()].cpu().numpy().view(np.uint16)
            got_v = vflat[torch.from_numpy(sl).cuda()].cpu().numpy().view(np.uint16)
            assert np.array_equal(got_k, kn_h[step][layer])
            assert np.array_equal(got_v, vn_h[step][layer])

    # sampled outputs against the oracle over history + appended rows
    pick = W.rng(4243)
    rows = [(0, 0), (S - 1, Hq - 1)] + [(int(pick.integers(S)), int(pick.integers(Hq))) for _ in range(SAMPLES - 2)]
    for step, (outs, _, lens) in enumerate(over):
        assert all(int(n) == hb.lengths[0] + step + 1 for n in lens)
        for layer in range(LAYERS):
            got = as_f64(outs[layer])
            for s, h in rows:
                kv = h // G
                kh = np.roll(hb.k_hist[s][:, kv], layer, axis=1)
                vh = np.roll(hb.v_hist[s][:, kv], layer, axis=1)
                kh = np.concatenate([kh] + [kn_h[t][layer][s, kv][None] for t in range(step + 1)])
                vh = np.concatenate([vh] + [vn_h[t][layer][s, kv][None] for t in range(step + 1)])
                ref = oatt.dense_decode_head(qs_h[step][layer][s, h], kh, vh, wl.scale)
                err = np.abs(got[s, h] - ref)
                assert np.all(err <= bf16_out_tol(ref, 1e-2)), (step, layer, s, h, float(err.max()))
