"""Host-only checks of the C ABI: the library builds and loads without a GPU,
exports every function ``include/mfa.h`` declares, and rejects malformed
descriptors before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libmfa():
    from decode_attention_08_b200 import build, mfa
    build.build()
    return mfa.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "mfa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mfa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("mfa_decode_attention", "mfa_query_proj"):
        assert required in names


def test_library_exports_every_declared_symbol(libmfa):
    from decode_attention_08_b200 import mfa
    for name in _declared_functions():
        assert hasattr(libmfa, name), f"libmfa.so does not export {name}"
    assert set(mfa.EXPORTS) >= set(_declared_functions())


def test_product_path_never_reaches_the_oracle(libmfa):
    """Neither the library nor the binding may link, import or call the oracle."""
    assert not hasattr(libmfa, "mfa_oracle_decode")
    pkg = os.path.join(ROOT, "decode_attention_08_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "mfa_oracle" not in text, f


def test_error_strings_and_version(libmfa):
    from decode_attention_08_b200 import mfa
    assert mfa.version() == 100
    for code, name in mfa.STATUS.items():
        assert mfa.error_string(code).startswith(name)


def test_null_and_malformed_descriptors_are_rejected_on_host(libmfa):
    from decode_attention_08_b200 import mfa
    T = mfa.MfaTensor
    null = ctypes.POINTER(T)()
    rc = libmfa.mfa_decode_attention(null, null, null, null, null, null, 0.0625, 0, None)
    assert rc == 1
    # a descriptor with a null data pointer
    d = T()
    d.data = None
    d.ndim = 3
    p = ctypes.pointer(d)
    assert libmfa.mfa_decode_attention_ex(p, p, p, null, p, p, 0.0625, 0, 1.0, 1.0, 0, null,
                                          None, 0, None) == 1
    assert libmfa.mfa_query_proj(null, null, null, null, None) == 1
    assert libmfa.mfa_kv_append(null, null, null, null, null, null, null, 0, 1.0, 1.0, None, 0,
                                None) == 1
    assert libmfa.mfa_output_proj(null, null, null, None, 0, None) == 1
    assert libmfa.mfa_lse_merge(null, null, null, null, None) == 1


def _fake(shape, dtype_code, addr=0x100000, strides=None):
    from decode_attention_08_b200 import mfa
    d = mfa.MfaTensor()
    d.data = addr
    d.dtype = dtype_code
    d.ndim = len(shape)
    st = strides
    if st is None:
        st, acc = [], 1
        for s in reversed(shape):
            st.insert(0, acc)
            acc *= s
    for i, (s, t) in enumerate(zip(shape, st)):
        d.shape[i] = s
        d.stride[i] = t
    return ctypes.pointer(d)


def test_shape_and_dtype_validation(libmfa):
    """Wrong heads/dims/dtypes fail validation before any CUDA call (fake, never
    dereferenced device addresses)."""
    null = ctypes.POINTER(__import__("decode_attention_08_b200.mfa",
                                     fromlist=["MfaTensor"]).MfaTensor)()
    B = 2
    q = _fake([B, 64, 256], 0)
    kv = _fake([B, 128, 256], 0)
    lens = _fake([B], 3)
    out = _fake([B, 64, 256], 1)
    f = libmfa.mfa_decode_attention
    assert f(_fake([B, 32, 256], 0), kv, kv, null, lens, out, 0.0625, 0, None) == 2   # H != 64
    assert f(_fake([B, 64, 128], 0), kv, kv, null, lens, out, 0.0625, 0, None) == 2   # d != 256
    assert f(_fake([B, 64, 256], 1), kv, kv, null, lens, out, 0.0625, 0, None) == 1   # q not bf16
    assert f(q, kv, _fake([B, 64, 256], 0), null, lens, out, 0.0625, 0, None) == 1    # k/v differ
    assert f(q, kv, kv, null, _fake([B + 1], 3), out, 0.0625, 0, None) == 1          # lens shape
    assert f(q, kv, kv, null, lens, _fake([B, 64, 256], 3), 0.0625, 0, None) == 1    # out dtype
    assert f(q, kv, kv, null, lens, out, 0.0625, 7, None) == 1                        # kv dtype
    assert f(q, kv, kv, null, lens, out, float("nan"), 0, None) == 1                  # scale NaN
    # misaligned token stride (not a multiple of 16 bytes)
    bad = _fake([B, 128, 256], 0, strides=[128 * 260, 260 + 1, 1])
    assert f(q, bad, bad, null, lens, out, 0.0625, 0, None) == 1
    # paged with an unsupported page size
    pt = _fake([B, 4], 3)
    pool = _fake([8, 48, 256], 0)
    assert f(q, pool, pool, pt, lens, out, 0.0625, 0, None) == 2
    # projection shape checks
    x = _fake([8, 7168], 0)
    wa = _fake([7168, 2048], 0)
    wb = _fake([2048, 16384], 0)
    qo = _fake([8, 16384], 0)
    g = libmfa.mfa_query_proj
    assert g(x, _fake([7000, 2048], 0), wb, qo, None) == 1
    assert g(_fake([129, 7168], 0), wa, wb, _fake([129, 16384], 0), None) == 2
    assert g(x, wa, wb, _fake([8, 16000], 0), None) == 1


def test_lse_merge_validation(libmfa):
    """Descriptor checks of mfa_lse_merge, before any CUDA call (fake addresses)."""
    null = ctypes.POINTER(__import__("decode_attention_08_b200.mfa",
                                     fromlist=["MfaTensor"]).MfaTensor)()
    S, B = 4, 3
    o = _fake([S, B, 64, 256], 1)
    lse = _fake([S, B, 64], 1)
    out = _fake([B, 64, 256], 0)
    f = libmfa.mfa_lse_merge
    assert f(_fake([S, B, 64, 256], 0), lse, out, null, None) == 1   # parts not f32
    assert f(_fake([S, B, 32, 256], 1), lse, out, null, None) == 2   # 32 heads
    assert f(o, _fake([S, B + 1, 64], 1), out, null, None) == 1      # lse shape
    assert f(o, lse, _fake([B, 64, 256], 3), null, None) == 1        # out dtype
    assert f(o, lse, out, _fake([B, 63], 1), None) == 1             # lse_out shape
    assert f(_fake([0, B, 64, 256], 1), _fake([0, B, 64], 1), out, null, None) == 1  # no parts
    misaligned = _fake([S, B, 64, 256], 1, strides=[B * 64 * 258, 64 * 258, 258, 1])
    assert f(misaligned, lse, out, null, None) == 1                  # float4 loads need 16 B
    assert f(o, lse, _fake([B, 64, 256], 0, addr=0x100004), null, None) == 1  # bf16 out 8 B


def test_workspace_size_is_zero_for_bad_arguments(libmfa):
    assert libmfa.mfa_decode_workspace_size(0, 0) == 0
    assert libmfa.mfa_decode_workspace_size(4, -1) == 0
    assert libmfa.mfa_query_proj_workspace_size(0, 7168, 2048) == 0
