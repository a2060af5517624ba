"""Unit tests of the causal multi-query attention kernels (tcgen05 and
plain-FMA) through the testing ABI, against the oracle's attention forward and
backward in float64 on the same bf16 inputs."""
import ctypes

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import lib  # noqa: E402

P = ctypes.c_void_p


def _bf16(x):
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def _run(B, T, H, nkv, hd, use_tc, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    Nqkv = (H + 2 * nkv) * hd
    qkv = _bf16(rng.standard_normal((B * T, Nqkv)) * scale)
    dO = _bf16(rng.standard_normal((B * T, H * hd)))
    qkv_d, dO_d = qkv.cuda(), dO.cuda()
    o = torch.full((B * T, H * hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    Tp = (T + 127) // 128 * 128  # softmax statistics are [B, H, T padded to 128]
    lse = torch.full((B * H * Tp,), float("nan"), dtype=torch.float32, device="cuda")
    dqkv = torch.full((B * T, Nqkv), float("nan"), dtype=torch.bfloat16, device="cuda")
    Dbuf = torch.full((2 * B * H * Tp,), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nws = lib().nc_test_attention_workspace_bytes(B, T, H, nkv, hd) if use_tc else 0
    # scratch starts as NaN bit patterns: every tile the kernels read must have been written
    ws = torch.full((max(nws // 2, 1),), float("nan"), dtype=torch.bfloat16, device="cuda")
    r = lib().nc_test_attention(B, T, H, nkv, hd, P(qkv_d.data_ptr()), P(o.data_ptr()), P(lse.data_ptr()),
                                P(dO_d.data_ptr()), P(dqkv.data_ptr()), P(Dbuf.data_ptr()), P(ws.data_ptr()), nws,
                                use_tc, P(status.data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    assert r == 0, r
    torch.cuda.synchronize()
    assert status.item() == 0
    q64 = qkv.double().numpy().reshape(B, T, H + 2 * nkv, hd)
    do64 = dO.double().numpy().reshape(B, T, H, hd)
    got_o = o.double().cpu().numpy().reshape(B, T, H, hd)
    got_d = dqkv.double().cpu().numpy().reshape(B, T, H + 2 * nkv, hd)
    for b in range(B):
        q, k, v = q64[b, :, :H], q64[b, :, H:H + nkv], q64[b, :, H + nkv:]
        ref_o = oracle.attention(q, k, v)
        dq, dk, dv = oracle.attention_backward(q, k, v, do64[b])
        for name, got, ref in (("o", got_o[b], ref_o), ("dq", got_d[b, :, :H], dq),
                               ("dk", got_d[b, :, H:H + nkv], dk), ("dv", got_d[b, :, H + nkv:], dv)):
            err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert err <= 1.5e-2, (name, b, err)


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("B,T,H,nkv", [(1, 128, 1, 1), (2, 300, 4, 1), (1, 513, 3, 1), (2, 256, 4, 2),
                                       (1, 1024, 2, 1), (3, 64, 2, 1)])
def test_tcgen05_attention(B, T, H, nkv, hd):
    _run(B, T, H, nkv, hd, 1, seed=T + H)


def test_tcgen05_attention_long_context():
    # the attention-heavy workload's sequence length (T = 8192, 64 query blocks), one
    # MQA pair of query heads; the oracle holds 8192 x 8192 float64 matrices per head
    _run(1, 8192, 2, 1, 128, 1, seed=8192)


def test_tcgen05_attention_sharp_softmax():
    # large scores: exercises the running-max rescale of the output
    _run(1, 640, 2, 1, 128, 1, seed=3, scale=4.0)


@pytest.mark.parametrize("hd", [16, 64])
def test_fma_attention(hd):
    _run(2, 150, 4, 1, hd, 0, seed=5)
