"""Launch overlap (programmatic dependent launch) leaves every result unchanged.

A decode step of several layers, each with its own pools, with the new token's
append folded in, is run twice from the same state: once with ordinary
launches and once with pkv_set_launch_overlap(1) for every layer after the
first (the first follows the plan kernel, whose output it reads).  Outputs and pools must be
bit-identical, and the outputs must match the float64 oracle; with 4 and with
16 grouped heads per KV head.
"""
import numpy as np
import pytest

import workloads as W
from oracle import attention as oatt
from tests.paged_batch import as_f64, device_batch, host_batch, torch_from_host

pytestmark = pytest.mark.gpu


def _step(pkv, torch, db, qs, kn, vn, slots, pools, scale, ws, out_dtype, overlap):
    outs = []
    for i, (kp, vp) in enumerate(pools):
        out = torch.empty(qs[i].shape, dtype=out_dtype, device="cuda")
        # the first layer follows the plan kernel, which writes what it reads first
        pkv.set_launch_overlap(overlap and i > 0)
        pkv.paged_decode_attn_append_run(qs[i], kn[i], vn[i], slots, kp, vp, db.tables, db.seq_lens, scale, out, ws)
        outs.append(out)
    pkv.set_launch_overlap(False)
    return outs


@pytest.mark.parametrize("heads", [None, (32, 2)], ids=["g4", "g16"])
def test_overlap_is_bit_identical_and_matches_oracle(heads):
    """g4: the 512-request workload's shapes (H_q 32, H_kv 8).  g16: 16 grouped
    heads per KV head, where each layer is two launches (the partition kernel
    and the merge of its split pieces), so a layer's partition kernel starts
    during the tail of the previous layer's merge launch."""
    import torch

    import paged_kv_cache_358_b200 as pkv

    wl = W.workload("mixed_512", block_size=16)
    lengths = [int(n) + 1 for n in wl.lengths[:96]]          # history + the new token
    if heads is not None:
        wl = W.DecodeWorkload("overlap_g16", 1, heads[0], heads[1], wl.head_dim, 16, "bf16", tuple(lengths),
                              pool_blocks=sum(-(-n // 16) for n in lengths) + 8, seed=23)
    hb = host_batch(wl, lengths=lengths, seed=21)
    db = device_batch(hb)
    S, Hq, Hkv, D, B = len(lengths), wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
    layers = 4
    g = W.rng(22)
    qs_h = [W.normal_bf16_bits(g, (S, Hq, D)) for _ in range(layers)]
    kn_h = [W.normal_bf16_bits(g, (S, Hkv, D)) for _ in range(layers)]
    vn_h = [W.normal_bf16_bits(g, (S, Hkv, D)) for _ in range(layers)]
    qs = [torch_from_host(x) for x in qs_h]
    kn = [torch_from_host(x) for x in kn_h]
    vn = [torch_from_host(x) for x in vn_h]
    pos = torch.tensor([n - 1 for n in lengths], dtype=torch.int32, device="cuda")
    slots = pkv.slot_mapping(db.tables, pos, B)
    base = [(db.k_pool.clone(), db.v_pool.clone()) for _ in range(layers)]
    ws = pkv.new_workspace(S, Hq, Hkv, D)
    results = []
    for on in (False, True):
        pools = [(k.clone(), v.clone()) for k, v in base]
        pkv.decode_plan(db.seq_lens, Hq, Hkv, D, pkv.BF16, ws)
        try:
            outs = _step(pkv, torch, db, qs, kn, vn, slots, pools, wl.scale, ws, torch.float32, on)
            outs2 = _step(pkv, torch, db, qs, kn, vn, slots, pools, wl.scale, ws, torch.float32, on)
        finally:
            pkv.set_launch_overlap(False)
        torch.cuda.synchronize()
        assert pkv.decode_status(ws) == 0
        results.append((outs, outs2, pools))
    (o_a, o2_a, p_a), (o_b, o2_b, p_b) = results
    for x, y in zip(o_a + o2_a, o_b + o2_b):
        assert torch.equal(x, y)
    for (ka, va), (kb, vb) in zip(p_a, p_b):
        assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
        assert torch.equal(va.view(torch.int16), vb.view(torch.int16))
    # the oracle: history with the appended row as its last token, per layer
    for layer in range(layers):
        got = as_f64(o_b[layer])
        for s in range(0, S, 7):
            kh = hb.k_hist[s].copy()
            vh = hb.v_hist[s].copy()
            kh[-1] = kn_h[layer][s]
            vh[-1] = vn_h[layer][s]
            ref = oatt.dense_decode(qs_h[layer][s], kh, vh, wl.scale)
            assert np.max(np.abs(got[s] - ref)) <= 1e-2
