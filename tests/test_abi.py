"""Host-side checks of the C ABI (no GPU needed): the library builds, loads and
exports every function include/sage2.h declares, and argument validation
returns its status codes before anything touches CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sage2.h")


@pytest.fixture(scope="module")
def L():
    from quantized_attention_04_b200 import build
    build.build()
    import quantized_attention_04_b200 as qa
    return qa.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sage2_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("sage2_attn_fwd", "sage2_smooth_quant_qk", "sage2_quant_v",
                 "sage2_attn_fwd_quantized", "sage2_debug_qk_s32", "sage2_workspace_bytes",
                 "sage2_check_device_error", "sage2_status_string",
                 # the variants (INT8 Q/K, V smoothing)
                 "sage2_attn_fwd_ex", "sage2_smooth_quant_qk_ex", "sage2_quant_v_ex",
                 "sage2_attn_fwd_quantized_ex", "sage2_debug_qk_s32_ex",
                 # packed variable-length sequences
                 "sage2_attn_fwd_varlen"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings(L):
    for s in range(7):
        assert L.sage2_status_string(s)
    assert L.sage2_status_string(99) == b"unknown status"


P = 0x10000  # 16-byte aligned fake address: never dereferenced by the checks below


def _attn(L, q=P, k=P, v=P, o=P, B=1, H=2, N=256, d=64, dt=0, odt=2, causal=0, sm=0.125):
    return L.sage2_attn_fwd(q, k, v, o, B, H, N, d, dt, odt, causal, sm, None)


def test_validation_codes(L):
    assert _attn(L, B=0) == 1
    assert _attn(L, N=0) == 1
    assert _attn(L, H=-1) == 1
    assert _attn(L, d=96) == 2
    assert _attn(L, d=256) == 2
    assert _attn(L, q=0) == 1
    assert _attn(L, o=0) == 1
    assert _attn(L, v=P + 8) == 3
    assert _attn(L, dt=2) == 1          # fp32 inputs are not a supported input dtype
    assert _attn(L, odt=3) == 1
    assert _attn(L, causal=2) == 1
    assert _attn(L, sm=0.0) == 1
    assert _attn(L, sm=float("nan")) == 1
    assert _attn(L, sm=float("inf")) == 1
    assert _attn(L, B=65536, H=1) == 2  # grid / 32-bit index limits
    assert _attn(L, B=1, H=1, N=2 ** 31 - 1) == 2


def test_validation_other_entries(L):
    z = [P] * 7
    assert L.sage2_smooth_quant_qk(P, P, 0, 1, 1, 0, 64, *z, None) == 1
    assert L.sage2_smooth_quant_qk(P, P, 0, 1, 1, 10, 80, *z, None) == 2
    assert L.sage2_smooth_quant_qk(P, P, 5, 1, 1, 10, 64, *z, None) == 1
    assert L.sage2_smooth_quant_qk(P, P, 0, 1, 1, 10, 64, P, P, P, P, P, 0, P, None) == 1
    assert L.sage2_smooth_quant_qk(P, P, 0, 1, 1, 10, 64, P, P, P, P, P + 4, P, P, None) == 3
    assert L.sage2_quant_v(P, 0, 1, 1, 10, 64, P, 0, None) == 1
    assert L.sage2_quant_v(P, 1, 1, 1, 10, 64, P + 1, P, None) == 3
    assert L.sage2_attn_fwd_quantized(P, P, P, P, P, P, P, P, 2, 1, 1, 10, 100, 0, 0.1, None) == 2
    assert L.sage2_attn_fwd_quantized(P, P, P, P, P, P, P, 0, 2, 1, 1, 10, 64, 0, 0.1, None) == 1
    assert L.sage2_debug_qk_s32(P, P, 1, 1, 10, 64, 0, None) == 1


def test_validation_variant_entries(L):
    def attn_ex(fmt=0, smooth=0, **kw):
        a = dict(q=P, k=P, v=P, o=P, B=1, H=2, N=256, d=64, dt=0, odt=2, causal=0, sm=0.125)
        a.update(kw)
        return L.sage2_attn_fwd_ex(a["q"], a["k"], a["v"], a["o"], a["B"], a["H"], a["N"], a["d"],
                                   a["dt"], a["odt"], a["causal"], a["sm"], fmt, smooth, None)
    assert attn_ex(fmt=3) == 1
    assert attn_ex(fmt=-1) == 1
    assert attn_ex(fmt=2, d=96) == 2               # packed INT4 is a valid format
    assert attn_ex(fmt=2, q=P + 4) == 3
    assert attn_ex(smooth=2) == 1
    assert attn_ex(fmt=1, d=96) == 2
    assert attn_ex(fmt=1, q=P + 4) == 3
    z = [P] * 7
    assert L.sage2_smooth_quant_qk_ex(P, P, 0, 1, 1, 10, 64, *z, 3, None) == 1
    assert L.sage2_smooth_quant_qk_ex(P, P, 0, 1, 1, 10, 64, *z, 0x100 | 3, None) == 1
    assert L.sage2_smooth_quant_qk_ex(P, P, 0, 1, 1, 10, 96, *z, 0x100 | 2, None) == 2
    assert L.sage2_smooth_quant_qk_ex(P, P, 0, 1, 1, 0, 64, *z, 1, None) == 1
    assert L.sage2_quant_v_ex(P, 0, 1, 1, 10, 64, P, P, P + 8, None) == 3     # misaligned v_mean
    assert L.sage2_quant_v_ex(P, 0, 1, 1, 10, 64, P, 0, P, None) == 1
    assert L.sage2_attn_fwd_quantized_ex(P, P, P, P, P, P, P, P, P, 2, 1, 1, 10, 64, 0, 0.1, 5,
                                         None) == 1
    assert L.sage2_attn_fwd_quantized_ex(P, P, P, P, P, P, P, P + 4, P, 2, 1, 1, 10, 64, 0, 0.1, 1,
                                         None) == 3
    assert L.sage2_debug_qk_s32_ex(P, P, 1, 1, 10, 64, 7, P, None) == 1
    assert L.sage2_debug_qk_s32_ex(P, P, 1, 1, 10, 64, 2, P, None) == 1   # packed: not here
    assert L.sage2_debug_qk_s32_ex(P, P, 1, 1, 10, 64, 1, 0, None) == 1


def test_validation_varlen(L):
    import ctypes
    def call(cu, S=None, H=2, T=None, d=64, **kw):
        arr = (ctypes.c_int * len(cu))(*cu)
        S = len(cu) - 1 if S is None else S
        T = cu[-1] if T is None else T
        a = dict(q=P, k=P, v=P, o=P, dt=0, odt=2, causal=0, sm=0.125, fmt=0, smooth=0)
        a.update(kw)
        return L.sage2_attn_fwd_varlen(a["q"], a["k"], a["v"], a["o"], arr, S, H, T, d, a["dt"],
                                       a["odt"], a["causal"], a["sm"], a["fmt"], a["smooth"], None)
    assert call([1, 5, 9]) == 1            # must start at 0
    assert call([0, 5, 3]) == 1            # must not decrease
    assert call([0, 5, 9], T=10) == 1      # must end at T
    assert call([0, 5, 9], S=0) == 1
    assert call([0, 5, 9], d=96) == 2
    assert call([0, 5, 9], fmt=4) == 1
    assert call([0, 5, 9], smooth=3) == 1
    assert call([0, 5, 9], q=P + 8) == 3
    assert call([0, 5, 9], causal=2) == 1
    assert L.sage2_attn_fwd_varlen(P, P, P, P, None, 2, 2, 9, 64, 0, 2, 0, 0.1, 0, 0, None) == 1


def test_workspace_bytes(L):
    def expect(B, H, N, d):
        up = lambda x: (x + 255) // 256 * 256
        Np = (N + 127) // 128 * 128
        NB = Np // 128
        BH = B * H
        parts = [BH * Np * d, BH * Np * d, BH * d * Np, BH * Np * 4, BH * Np * 4,
                 BH * NB * d * 4, BH * d * 4, BH * NB * Np * 4, BH * d * 4, BH * NB * d * 4,
                 BH * d * 4, 3 * BH * ((NB + 127) // 128) * 128 * d * 2, BH * d * 4,
                 2 * BH * 4]
        return sum(up(p) for p in parts)
    for shape in [(1, 2, 256, 64), (2, 8, 2048, 128), (1, 24, 17776, 64), (1, 1, 1, 128)]:
        assert L.sage2_workspace_bytes(*shape) == expect(*shape)
    assert L.sage2_workspace_bytes(0, 1, 1, 64) == 0
    assert L.sage2_workspace_bytes(1, 1, 1, 32) == 0
