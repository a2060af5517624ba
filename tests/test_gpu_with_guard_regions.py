"""Guard regions around the outputs of the step and of the GEMM and attention
kernels: every output buffer sits inside a larger one filled with a canary
value, and after the run every byte outside the documented extent must still
hold the canary.  (Bounds checking without compute-sanitizer.)"""
import ctypes

import numpy as np
import pytest

import synth
from harness import to_device_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import Model, lib  # noqa: E402

P = ctypes.c_void_p
CANARY = -7777.0
PAD = 4096  # elements of guard on each side (16-byte aligned for every dtype used)


def _guarded(n, dtype):
    buf = torch.full((n + 2 * PAD,), CANARY, dtype=dtype, device="cuda")
    return buf, buf[PAD:PAD + n]


def _guard_intact(buf, n):
    ref = torch.full((PAD,), CANARY, dtype=buf.dtype, device="cuda")
    return torch.equal(buf[:PAD], ref) and torch.equal(buf[PAD + n:], ref)


@pytest.mark.parametrize("B,T", [(2, 32), (3, 37)])
def test_step_writes_only_its_outputs(B, T):
    cfg = synth.WORKLOADS["tiny"].model
    bits, w = synth.make_weights(cfg, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(synth.Workload("case", cfg, T, B, "uniform"), seed=1)
    m = Model(cfg, "bf16")
    n = m.num_params()
    gbuf, grads = _guarded(n, torch.float32)
    lbuf, loss = _guarded(1, torch.float32)
    wsb = m.workspace_bytes(B, T)
    wbuf = torch.full((wsb + 2 * PAD,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = wbuf[PAD:PAD + wsb]
    m.forward_backward(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda(),
                       to_device_weights(bits, w, "bf16"), grads, loss, ws)
    assert m.check() == 0
    assert _guard_intact(gbuf, n) and _guard_intact(lbuf, 1)
    ref = torch.full((PAD,), 0xA5, dtype=torch.uint8, device="cuda")
    assert torch.equal(wbuf[:PAD], ref) and torch.equal(wbuf[PAD + wsb:], ref)
    assert torch.isfinite(grads).all() and torch.isfinite(loss).all()


@pytest.mark.parametrize("M,N,K", [(200, 72, 136), (384, 264, 192)])
@pytest.mark.parametrize("epi,c_bf16", [(0, False), (1, False), (0, True)])
def test_gemm_writes_only_its_tile(M, N, K, epi, c_bf16):
    gen = torch.Generator().manual_seed(M + N + K + epi)
    A = torch.randn(M, K, generator=gen).to(torch.bfloat16).cuda()
    B = torch.randn(N, K, generator=gen).to(torch.bfloat16).cuda()
    ldc = N + 8  # padded rows: columns N..ldc-1 must stay untouched
    cdt = torch.bfloat16 if c_bf16 else torch.float32
    rows = M + 2  # two guard rows after the output
    cbuf, _ = _guarded(rows * ldc, cdt)
    C = cbuf[PAD:PAD + rows * ldc].view(rows, ldc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = lib().nc_test_gemm(M, N, K, 1, P(A.data_ptr()), K, 1, P(B.data_ptr()), K, 1, epi, P(C.data_ptr()), ldc,
                           int(c_bf16), P(0), 0, P(0), 0, ctypes.c_float(15.0), 1, P(0), 0,
                           P(status.data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    assert r == 0, r
    torch.cuda.synchronize()
    assert status.item() == 0
    assert _guard_intact(cbuf, rows * ldc)
    canary = torch.full((1,), CANARY, dtype=cdt, device="cuda")
    assert torch.equal(C[:M, N:], canary.expand(M, ldc - N))
    assert torch.equal(C[M:, :], canary.expand(rows - M, ldc))
    # the tile itself was written
    assert not torch.equal(C[:M, :N], canary.expand(M, N))


@pytest.mark.parametrize("T,hd", [(300, 128), (129, 64)])
def test_attention_writes_only_its_outputs(T, hd):
    B, H, nkv = 2, 3, 1
    gen = torch.Generator().manual_seed(T + hd)
    nq = (H + 2 * nkv) * hd
    qkv = torch.randn(B * T * nq, generator=gen).to(torch.bfloat16).cuda()
    dO = torch.randn(B * T * H * hd, generator=gen).to(torch.bfloat16).cuda()
    Tp = (T + 127) // 128 * 128
    obuf, o = _guarded(B * T * H * hd, torch.bfloat16)
    lbuf, lse = _guarded(B * H * Tp, torch.float32)
    dbuf, dq = _guarded(B * T * nq, torch.bfloat16)
    Dbb, Dbuf = _guarded(2 * B * H * Tp, torch.float32)
    nws = lib().nc_test_attention_workspace_bytes(B, T, H, nkv, hd)
    wbuf, ws = _guarded(nws // 2, torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = lib().nc_test_attention(B, T, H, nkv, hd, P(qkv.data_ptr()), P(o.data_ptr()), P(lse.data_ptr()),
                                P(dO.data_ptr()), P(dq.data_ptr()), P(Dbuf.data_ptr()), P(ws.data_ptr()), nws, 1,
                                P(status.data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    assert r == 0, r
    torch.cuda.synchronize()
    assert status.item() == 0
    assert _guard_intact(obuf, B * T * H * hd) and _guard_intact(lbuf, B * H * Tp)
    assert _guard_intact(dbuf, B * T * nq) and _guard_intact(Dbb, 2 * B * H * Tp)
    assert _guard_intact(wbuf, nws // 2)
    assert torch.isfinite(o.float()).all() and torch.isfinite(dq.float()).all()
    assert np.isfinite(lse.view(B, H, Tp)[:, :, :T].cpu().numpy()).all()
