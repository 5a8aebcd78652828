"""The C-ABI library loads on a machine without a GPU and exports every entry
point that include/pkv.h declares (no compute call is made here)."""
import ctypes
import os
import re

from tests.conftest import ROOT


def _declared():
    with open(os.path.join(ROOT, "include", "pkv.h"), encoding="utf-8") as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("pkv_paged_decode_attn", "pkv_kv_append", "pkv_block_copy", "pkv_slot_mapping",
                     "pkv_alloc_create", "pkv_alloc_append", "pkv_alloc_free_seq", "pkv_alloc_check"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import paged_kv_cache_358_b200 as pkv

    L = pkv.lib()
    missing = [n for n in _declared() if not hasattr(L, n)]
    assert missing == []
    assert L.pkv_version().decode().startswith("pkv ")
    assert L.pkv_status_string(1).decode() == "no free blocks"


def test_python_binding_is_thin():
    """The binding holds no kernels or CPU fallback: only ctypes marshalling."""
    import paged_kv_cache_358_b200 as pkv

    src = open(pkv.__file__, encoding="utf-8").read()
    assert "import oracle" not in src and "from oracle" not in src
    for banned in ("torch.softmax", ".softmax(", "nn.functional", "einsum(", "matmul(", "torch.exp("):
        assert banned not in src, banned
