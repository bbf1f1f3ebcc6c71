"""GPU: the host-buffer pipeline (vc_attn_run_host) gives exactly the output of
the three device calls on the whole problem, for ragged head chunks, B > 1,
both residual formats, and pinned or pageable host memory."""
import pytest
import torch

from bit_fp8_attention_prep_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    from bit_fp8_attention_prep_b200 import build, vc_attn
    build.build()
    vc_attn.load()
    return vc_attn


def _device_reference(va, Q, K, V, fmt, dtype):
    B, S, H, _ = Q.shape
    plan = va.Plan(B, S, H, dtype=dtype, fmt=fmt)
    o = plan.run(Q.cuda(), K.cuda(), V.cuda()).clone()
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    return o.cpu()


@pytest.mark.parametrize("fmt,chunk,pinned,dtype", [
    ("e4m3", 2, True, torch.bfloat16),     # chunks of 2, 1 heads per batch entry
    ("e4m3", 3, False, torch.float16),     # one chunk per batch entry, pageable memory
    ("nvfp4", 1, True, torch.bfloat16),
])
def test_run_host_matches_device_path(va, fmt, chunk, pinned, dtype):
    Q, K, V = synth.make_qkv(2, 1000, 3, recipe="mixture", seed=3, dtype=dtype)
    ref = _device_reference(va, Q, K, V, fmt, dtype)
    hq, hk, hv = (X.pin_memory() if pinned else X.clone() for X in (Q, K, V))
    ho = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16)
    ho = ho.pin_memory() if pinned else ho
    hp = va.HostPlan(2, 1000, 3, dtype=dtype, fmt=fmt, head_chunk=chunk)
    for _ in range(2):                      # the second call reuses the workspace and the copy streams
        ho.fill_(float("nan"))
        hp.run(hq, hk, hv, ho)
        torch.cuda.current_stream().synchronize()
        assert int(hp.status.item()) == 0
        assert torch.equal(ho.view(torch.int16), ref.view(torch.int16))


def test_run_host_rejects_device_tensors(va):
    hp = va.HostPlan(1, 256, 2, head_chunk=1)
    x = torch.zeros(1, 256, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        hp.run(x, x, x, torch.empty(1, 256, 2, 128, dtype=torch.bfloat16))
