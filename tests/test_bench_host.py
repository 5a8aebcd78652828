"""Host-side pieces of bench.py that need no GPU: the algorithmic byte count,
the traffic file and the peak lookup."""
import os
import types

import numpy as np

import bench


def _dummy(S=32, Hq=32, Hkv=8, D=128, L=32, B=16):
    return types.SimpleNamespace(S=S, Hq=Hq, Hkv=Hkv, D=D, L=L, B=B)


def test_step_bytes_count_each_history_slot_once_per_kv_head():
    d = _dummy()
    lens = np.full(32, 4097, dtype=np.int64)
    got = bench.DecodeStep.bytes_of_step(d, lens, 0)
    kv = 32 * 4097 * 8 * 128 * 2 * 2                     # K and V, bf16, once per KV head
    qo = 32 * 32 * 128 * 2 * 2                           # q read, out written
    app = 32 * 8 * 128 * 2 * 2 * 2                       # new K/V rows read and written
    meta = 4 * 32 * (-(-4097 // 16)) + 4 * 32            # table entries and lengths
    assert got == 32 * (kv + qo + app + meta) + 8 * 32   # + slots per request
    # the 16 GiB lower bound of the pages at 4096 tokens is contained in it
    assert 32 * 32 * 4096 * 8 * 128 * 2 * 2 == 16 * 2 ** 30


def test_copy_on_write_bytes_count_the_valid_rows_per_layer():
    """A copy-on-write moves n_valid = n mod B rows of K and V (read and written)
    in every layer, not the whole block: three copies of 8, 1 and 15 rows."""
    d = _dummy()
    lens = np.full(32, 100, dtype=np.int64)
    base = bench.DecodeStep.bytes_of_step(d, lens, 0)
    with_cow = bench.DecodeStep.bytes_of_step(d, lens, 8 + 1 + 15)
    row = 8 * 128 * 2                                   # one token of one layer's K (or V) pool
    assert with_cow - base == 32 * (8 + 1 + 15) * row * 2 * 2
    assert with_cow - base < 32 * 3 * 16 * row * 2 * 2  # less than three whole blocks


def test_step_stats_are_order_statistics():
    x = [3.0, 1.0, 2.0, 10.0, 4.0]
    st = bench.step_stats(x)
    assert st["median"] == 3.0 and st["n"] == 5
    assert st["p10"] == np.percentile(x, 10) and st["p90"] == np.percentile(x, 90)
    assert st["mean"] == 4.0


def test_traffic_file_is_read_by_key():
    path = os.path.join(bench.ROOT, "profiles", "traffic.txt")
    value = bench.read_traffic("paged_decode_attn_teaching_32x4096_bytes_per_launch")
    if os.path.exists(path):
        assert value is not None and 5.0e8 < value < 6.0e8    # one launch of the 32 x 4096 layer
    else:
        assert value is None
    assert bench.read_traffic("no_such_key") is None


def test_peak_is_measured_or_the_fallback():
    peak, kind = bench.peaks()
    assert kind in ("measured", "fallback")
    if kind == "fallback":
        assert peak == bench.FALLBACK_HBM_GBS
    assert 1000.0 < peak < 10000.0
