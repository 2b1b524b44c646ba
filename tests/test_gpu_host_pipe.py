"""The host-buffer entry (sage2_attn_fwd_host): chunks of heads copied in,
run and copied back on library streams.  Per-head arithmetic is the device
path's, so the result must equal sage2_attn_fwd bit for bit (pinned and
pageable host memory, several chunks and a ragged last chunk)."""
import pytest
import torch

from quantized_attention_04_b200.inputs import CONFIGS, Config, Dist, make_qkv
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qa():
    from quantized_attention_04_b200 import build
    build.build()
    import quantized_attention_04_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


CASES = [
    CONFIGS["C2"],
    Config("host_many_heads", 3, 7, 4000, 64, True, "fp16", q=Dist(1.0), k=Dist(3.0), v=Dist(2.0),
           index=70),
    # 4 MB heads: 4 heads per 48 MB chunk, so 5 chunks (the last one of 2 heads)
    # on the 4 library streams, the fifth reusing the first stream's buffers
    Config("host_chunks", 1, 18, 16384, 128, True, "bf16", q=Dist(1.0), k=Dist(3.0), v=Dist(2.0),
           index=71),
]


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_host_entry_equals_device_entry(qa, cfg, pinned):
    q, k, v = make_qkv(cfg)
    sm = P.default_scale(cfg.d)
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty(q.shape, dtype=torch.float32)
    if pinned:
        oh = oh.pin_memory()
    qa.sage2_attn_fwd_host(q, k, v, oh, causal=cfg.causal, sm_scale=sm)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    od = qa.sage2_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=cfg.causal, sm_scale=sm,
                           out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(oh, od.cpu())


def test_host_entry_packed_int4_equals_device_entry(qa):
    """The host-buffer entry with INT4 payloads stored two per byte equals the
    device entry (INT4 codes) bit for bit."""
    cfg = CASES[1]
    q, k, v = make_qkv(cfg)
    sm = P.default_scale(cfg.d)
    oh = torch.empty(q.shape, dtype=torch.float32).pin_memory()
    qa.sage2_attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), oh, causal=cfg.causal,
                           sm_scale=sm, packed=True)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    od = qa.sage2_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=cfg.causal, sm_scale=sm,
                           out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(oh, od.cpu())
