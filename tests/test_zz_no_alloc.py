"""The allocation-free weight-gradient GEMM (nc_gemm_wgrad_noalloc), for
callers that cannot allocate device memory, checked against the regular GEMM
entry point on two calls in a row.  This file is collected last on purpose."""
import ctypes

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import lib  # noqa: E402
from bwd_step_b200 import _lib  # noqa: E402

P = ctypes.c_void_p


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def _regular(rows, n_out, n_in, dy, x, dw, accumulate, status):
    scratch = torch.empty(8 * 4 * n_out * n_in, dtype=torch.uint8, device="cuda")
    r = lib().nc_test_gemm(n_out, n_in, rows, 1, P(dy.data_ptr()), n_out, 0, P(x.data_ptr()), n_in, 0,
                           1 if accumulate else 0, P(dw.data_ptr()), n_in, 0, P(0), 0, P(0), 0, ctypes.c_float(1.0),
                           1, P(scratch.data_ptr()), scratch.numel(), P(status.data_ptr()), _stream())
    assert r == 0, r


def _noalloc(rows, n_out, n_in, dy, x, dw, accumulate, status):
    r = lib().nc_gemm_wgrad_noalloc(rows, n_out, n_in, P(dy.data_ptr()), n_out, P(x.data_ptr()), n_in,
                                    P(dw.data_ptr()), 1 if accumulate else 0, P(status.data_ptr()), _stream())
    assert r == 0, r


@pytest.mark.parametrize("rows,n_out,n_in,accumulate", [(8192, 1280, 1280, False), (4096, 512, 1536, True)])
def test_two_calls_match_regular_entry_point(rows, n_out, n_in, accumulate):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(rows + n_in)
    for call in range(2):
        dy = torch.randn(rows, n_out, device="cuda", generator=g).to(torch.bfloat16)
        x = torch.randn(rows, n_in, device="cuda", generator=g).to(torch.bfloat16)
        init = torch.randn(n_out, n_in, device="cuda", generator=g)
        ref = init.clone()
        got = init.clone()
        _regular(rows, n_out, n_in, dy, x, ref, accumulate, status)
        _noalloc(rows, n_out, n_in, dy, x, got, accumulate, status)
        torch.cuda.synchronize()
        assert status.item() == 0
        err = (got - ref).norm() / ref.norm()
        assert err <= 2e-6, (call, float(err))


def test_rejects_results_larger_than_the_static_array():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    n = 4096  # 4096 x 4096 fp32 x 2 partials = 128 MiB > 64 MiB
    dy = torch.zeros(64, n, dtype=torch.bfloat16, device="cuda")
    dw = torch.zeros(n, n, dtype=torch.float32, device="cuda")
    r = lib().nc_gemm_wgrad_noalloc(64, n, n, P(dy.data_ptr()), n, P(dy.data_ptr()), n, P(dw.data_ptr()), 0,
                                    P(status.data_ptr()), _stream())
    assert r == _lib.NC_ERR_UNSUPPORTED_SHAPE


def test_rejects_misaligned_buffers_before_launching():
    """dw one float past a 16-byte boundary (a torch view at an odd offset) is
    refused with NC_ERR_INVALID_ARG; nothing runs, so its contents stay."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows, n = 4096, 256
    dy = torch.ones(rows, n, dtype=torch.bfloat16, device="cuda")
    buf = torch.full((n * n + 1,), 7.0, dtype=torch.float32, device="cuda")
    dw = buf[1:]
    r = lib().nc_gemm_wgrad_noalloc(rows, n, n, P(dy.data_ptr()), n, P(dy.data_ptr()), n, P(dw.data_ptr()), 0,
                                    P(status.data_ptr()), _stream())
    assert r == _lib.NC_ERR_INVALID_ARG
    r = lib().nc_gemm_wgrad_noalloc(rows, n, n, P(dy.data_ptr() + 2), n, P(dy.data_ptr()), n,
                                    P(buf.data_ptr()), 0, P(status.data_ptr()), _stream())
    assert r == _lib.NC_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.all(buf == 7.0) and status.item() == 0
