"""CPU checks of the boundary: the library loads and exports every symbol
that include/mk.h declares; host-side argument validation."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    from persistent_decode_megakernel_sm_b200 import mk
    lib = ctypes.CDLL(mk.LIB_PATH)
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(mk.EXPORTS) == names


def test_binding_is_marshalling_only():
    """The Python binding holds no arithmetic: no numpy, no torch math."""
    src = open(os.path.join(ROOT, "persistent_decode_megakernel_sm_b200", "mk.py")).read()
    assert "import numpy" not in src
    assert "import oracle" not in src and "from oracle" not in src
    for bad in ("torch.matmul", "softmax", "@", "einsum"):
        assert bad not in src.split('"""', 2)[2], bad


def test_product_never_imports_oracle():
    pkg = os.path.join(ROOT, "persistent_decode_megakernel_sm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cpp")):
                s = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in s and "from oracle" not in s and "oracle.c" not in s, f


@pytest.mark.parametrize("bad", [
    dict(hidden=100), dict(head_dim=96), dict(n_q_heads=6, n_kv_heads=4), dict(ffn=0), dict(max_batch=9),
])
def test_create_rejects_bad_shapes_on_host(bad):
    from persistent_decode_megakernel_sm_b200 import mk
    d = mk.mk_model_desc(layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=1024, vocab=4096,
                         rope_theta=1e4, rms_eps=1e-6, max_batch=8, max_ctx=160)
    for k, v in bad.items():
        setattr(d, k, v)
    with pytest.raises(mk.MkError) as e:
        mk.mk_create(d, 0)
    assert e.value.code == mk.MK_ERR_INVALID
    # a failed create returns no handle: the reason is read with a null handle
    assert mk.lib.mk_last_error(None).startswith(b"invalid model description: ")


def test_null_handle_calls_fail_cleanly():
    from persistent_decode_megakernel_sm_b200 import mk
    assert mk.lib.mk_decode_step(None, None, None, 1, None, None, None, None) == mk.MK_ERR_INVALID
    assert mk.lib.mk_sync_status(None) == mk.MK_ERR_INVALID
    assert isinstance(mk.lib.mk_last_error(None), bytes)
