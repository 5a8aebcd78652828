"""Argument checks of the C ABI's KV-cache operations, on the CPU.

`pkv_kv_append`, `pkv_block_copy`, `pkv_swap_blocks` and `pkv_slot_mapping`
check every argument before they launch anything, and return PKV_OK at once
when there is nothing to do (no token, copy or block).  Each call below
either breaks one check or has nothing to do, so none of them reaches a
launch or touches a pointer: the pointers are bare addresses, some of them
deliberately misaligned.  (The decode calls first read the device's SM
count to size their workers, so their argument checks are exercised by the
`-m gpu` tests.)
"""
import ctypes

import pytest

import paged_kv_cache_358_b200 as pkv

OK, INVALID = pkv.Status.OK, pkv.Status.INVALID
A, B_, C, D_ = 0x100000, 0x200000, 0x300000, 0x400000    # 16-byte aligned addresses (never dereferenced)
MIS = 0x500008                                            # 8-byte aligned only


def _ptrs(*addrs):
    return (ctypes.c_void_p * len(addrs))(*addrs)


def _append(k=A, v=B_, slots=C, n=4, kp=D_, vp=D_ + 0x1000, Hkv=8, D=128, B=16, N=64, dtype=pkv.BF16):
    return pkv.lib().pkv_kv_append(k, v, slots, n, kp, vp, Hkv, D, B, N, dtype, None)


@pytest.mark.parametrize("kw", [
    dict(dtype=7), dict(n=-1), dict(Hkv=0), dict(D=0), dict(N=-1),
    dict(B=24), dict(B=0), dict(B=2048),
    dict(Hkv=1, D=4),                  # 8-byte rows: not a multiple of 16 bytes
    dict(k=None), dict(slots=None), dict(vp=None),
    dict(k=MIS), dict(kp=MIS),
])
def test_kv_append_refuses(kw):
    assert _append(**kw) == INVALID


def test_kv_append_with_no_token_does_nothing():
    assert _append(n=0, k=None, v=None, slots=None, kp=None, vp=None) == OK


def _copy(kps=(A,), vps=(B_,), L=None, copies=C, n=2, Hkv=8, D=128, B=16, N=64, dtype=pkv.BF16):
    L = (len(kps) if kps is not None else 1) if L is None else L
    kp = _ptrs(*kps) if kps is not None else None
    vp = _ptrs(*vps) if vps is not None else None
    return pkv.lib().pkv_block_copy(kp, vp, L, copies, n, Hkv, D, B, N, dtype, None)


@pytest.mark.parametrize("kw", [
    dict(L=0), dict(L=129, kps=(A,) * 129, vps=(B_,) * 129), dict(n=-1), dict(B=3), dict(dtype=-1),
    dict(Hkv=1, D=4), dict(copies=None), dict(kps=None),
    dict(kps=(A, MIS), vps=(B_, B_ + 0x1000)),   # the second layer's K pool misaligned
    dict(kps=(A, None), vps=(B_, B_ + 0x1000)),
])
def test_block_copy_refuses(kw):
    assert _copy(**kw) == INVALID


def test_block_copy_with_no_copy_does_nothing():
    assert _copy(n=0, copies=None, kps=None, vps=None, L=1) == OK


def _swap(kps=(A,), vps=(B_,), blocks=C, n=2, host=D_, to_host=1, Hkv=8, D=128, B=16, N=64, dtype=pkv.BF16):
    kp = _ptrs(*kps) if kps is not None else None
    vp = _ptrs(*vps) if vps is not None else None
    return pkv.lib().pkv_swap_blocks(kp, vp, len(kps or (A,)), blocks, n, host, to_host, Hkv, D, B, N, dtype,
                                     None)


@pytest.mark.parametrize("kw", [
    dict(to_host=2), dict(n=-1), dict(B=12), dict(N=-3), dict(host=None), dict(host=MIS),
    dict(blocks=None), dict(B=1, Hkv=1, D=4),   # 8-byte blocks
    dict(kps=(MIS,)),
])
def test_swap_blocks_refuses(kw):
    assert _swap(**kw) == INVALID


def test_swap_blocks_with_no_block_does_nothing():
    assert _swap(n=0, blocks=None, host=None, kps=None, vps=None) == OK


def _slots(tables=A, max_blocks=8, rows=None, positions=B_, n=3, B=16, out=C):
    return pkv.lib().pkv_slot_mapping(tables, max_blocks, rows, positions, n, B, out, None)


@pytest.mark.parametrize("kw", [
    dict(n=-1), dict(max_blocks=-1), dict(B=0), dict(B=-16),
    dict(tables=None), dict(positions=None), dict(out=None),
])
def test_slot_mapping_refuses(kw):
    assert _slots(**kw) == INVALID


def test_slot_mapping_with_no_token_does_nothing():
    assert _slots(n=0, tables=None, positions=None, out=None) == OK
