"""The allocation-free entry point, sage2_attn_fwd_noalloc.

It exists for callers that must not have a library allocate device memory
while they run (hosts that forbid allocator calls after start-up, frameworks
that account for every device byte through their own allocator): it runs the
same kernels as sage2_attn_fwd with its scratch in one fixed device array.
These tests call it through the C ABI and compare it with sage2_attn_fwd, the
pooled entry point: both run the same deterministic kernels in the same order,
so the outputs must be identical bit for bit.  Two calls
run back to back, the second one smaller and with another head dimension and
dtype, so that it reads scratch left over by the first.  This file is named to
be collected last.
"""
import ctypes
import math

import pytest
import torch

from quantized_attention_04_b200.inputs import Config, Dist, make_qkv

SAGE2_ERR_TOO_LARGE = 7
_P = ctypes.c_void_p


def _lib():
    from quantized_attention_04_b200 import build
    build.build()
    import quantized_attention_04_b200 as qa
    return qa, qa.lib()


def _noalloc(L, q, k, v, o, causal, sm, stream):
    B, H, N, d = q.shape
    dt = {torch.float16: 0, torch.bfloat16: 1}[q.dtype]
    odt = {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2}[o.dtype]
    return L.sage2_attn_fwd_noalloc(_P(q.data_ptr()), _P(k.data_ptr()), _P(v.data_ptr()),
                                    _P(o.data_ptr()), B, H, N, d, dt, odt, int(causal),
                                    float(sm), _P(stream))


def test_noalloc_rejects_problems_beyond_its_buffer():
    """Rejected on the host, before anything touches a device."""
    _, L = _lib()
    big = L.sage2_workspace_bytes(1, 64, 32768, 128)
    assert big > 64 * 2 ** 20
    st = L.sage2_attn_fwd_noalloc(_P(0x10000), _P(0x10000), _P(0x10000), _P(0x10000),
                                  1, 64, 32768, 128, 1, 1, 1, 0.088, None)
    assert st == SAGE2_ERR_TOO_LARGE
    assert b"no-allocation" in L.sage2_status_string(SAGE2_ERR_TOO_LARGE)


@pytest.mark.gpu
def test_noalloc_matches_pooled_entry_on_two_calls_in_a_row():
    qa, L = _lib()
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    cfgs = [
        Config("noalloc_a", 2, 4, 1000, 128, True, "bf16",
               q=Dist(1.0), k=Dist(3.0, outliers=2, outlier_scale=8.0), v=Dist(1.0), index=40),
        Config("noalloc_b", 1, 3, 300, 64, False, "fp16",
               q=Dist(2.0), k=Dist(4.0), v=Dist(0.5), index=41),
    ]
    stream = torch.cuda.current_stream().cuda_stream
    for cfg in cfgs:
        q, k, v = (t.cuda() for t in make_qkv(cfg))
        sm = 1.0 / math.sqrt(cfg.d)
        o_free = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(L, q, k, v, o_free, cfg.causal, sm, stream) == 0
        o_pool = qa.sage2_attn_fwd(q, k, v, causal=cfg.causal, sm_scale=sm,
                                   out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert qa.sage2_check_device_error() == 0
        assert torch.equal(o_free, o_pool), cfg.name
