"""Unit tests of the tcgen05 GEMM (and the FMA GEMM) through the testing ABI:
every operand layout, every fused epilogue, ragged tails, split-K, against a
float64 product of the same bf16 inputs."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import lib  # noqa: E402

P = ctypes.c_void_p


def _operand(R, K, kmajor, gen, scale=1.0):
    x = (torch.randn(R, K, generator=gen) * scale).to(torch.bfloat16)
    stored = x if kmajor else x.t().contiguous()
    return x.double(), stored.cuda(), (K if kmajor else R)


def _run(M, N, K, ak, bk, epi, c_bf16, use_tc=1, seed=0, scale=1.0, scratch_mb=0, c_offset=0, tol=None):
    gen = torch.Generator().manual_seed(seed)
    A64, A, lda = _operand(M, K, ak, gen, scale)
    B64, B, ldb = _operand(N, K, bk, gen, scale)
    acc = A64 @ B64.t()
    cdt = torch.bfloat16 if c_bf16 else torch.float32
    C0 = torch.randn(M, N, generator=gen)
    # c_offset > 0 places C that many elements into a larger buffer (a view
    # whose base is not 16-byte aligned)
    Cbuf = torch.zeros(M * N + c_offset, dtype=cdt, device="cuda")
    C = Cbuf[c_offset:].view(M, N)
    C.copy_(C0.to(cdt))
    C2 = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    aux = torch.rand(M, N, generator=gen).to(torch.bfloat16)
    auxd = aux.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scratch = torch.empty(scratch_mb << 20, dtype=torch.uint8, device="cuda") if scratch_mb else None
    r = lib().nc_test_gemm(M, N, K, 1, P(A.data_ptr()), lda, int(ak), P(B.data_ptr()), ldb, int(bk), epi,
                           P(C.data_ptr()), N, int(c_bf16), P(C2.data_ptr()), N, P(auxd.data_ptr()), N,
                           ctypes.c_float(15.0), use_tc, P(scratch.data_ptr() if scratch is not None else 0),
                           scratch.numel() if scratch is not None else 0, P(status.data_ptr()),
                           P(torch.cuda.current_stream().cuda_stream))
    assert r == 0, r
    torch.cuda.synchronize()
    assert status.item() == 0
    if epi == 0:
        exp = acc
    elif epi == 1:
        exp = C0.double() + acc
    elif epi == 2:
        exp = torch.relu(acc) ** 2
        got2 = C2.double().cpu()
        _close(got2, torch.relu(acc), True, tol)
    elif epi == 3:
        exp = acc * 2 * aux.double()
    else:
        exp = 15.0 * torch.tanh(acc / 15.0)
    _close(C.double().cpu(), exp, c_bf16, tol)


def _close(got, exp, bf, tol=None):
    err = (got - exp).norm() / max(exp.norm(), 1e-30)
    assert err <= (tol or (4e-3 if bf else 2e-6)), float(err)


@pytest.mark.parametrize("ak,bk", [(True, True), (True, False), (False, False), (False, True)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (384, 512, 192), (200, 72, 136), (64, 96, 64),
                                   (1000, 776, 520)])
def test_layouts_and_tails(ak, bk, M, N, K):
    _run(M, N, K, ak, bk, 0, False, seed=M + N + K)


@pytest.mark.parametrize("epi,c_bf16", [(0, True), (1, False), (2, True), (3, True), (4, False), (4, True)])
def test_epilogues(epi, c_bf16):
    scale = 3.0 if epi == 4 else 1.0
    _run(520, 776, 328, True, True, epi, c_bf16, scale=scale, seed=epi)
    _run(264, 520, 200, True, False, epi, c_bf16, scale=scale, seed=10 + epi)


@pytest.mark.parametrize("ak,bk", [(False, False), (True, False)])
def test_split_k(ak, bk):
    # 2 x 1 output tiles with a long reduction: split over K, reduced in order
    _run(256, 256, 8192, ak, bk, 0, False, scratch_mb=64, seed=3)
    _run(256, 256, 8192, ak, bk, 1, False, scratch_mb=64, seed=4)


@pytest.mark.parametrize("M,N", [(896, 768), (200, 520), (1000, 264)])
def test_split_k_ragged_rows(M, N):
    # M not a multiple of the tile height: the last tile's extra rows must not
    # spill into the next split's partial sums
    _run(M, N, 4096, False, False, 0, False, scratch_mb=128, seed=M)
    _run(M, N, 4096, False, False, 1, False, scratch_mb=128, seed=M + 1)


@pytest.mark.parametrize("epi", [0, 1])
def test_split_k_candidate_with_unaligned_output(epi):
    # a shape that takes split-K, with C one float past a 16-byte boundary: the
    # vectorised split-K reduction must not be used (it would be a misaligned
    # access); the GEMM still runs, on the single-pass epilogue, whose one
    # 8192-long fp32 accumulation is looser than a sum of split partials
    _run(256, 256, 8192, False, False, epi, False, scratch_mb=64, seed=11 + epi, c_offset=1, tol=2e-5)


def test_fma_gemm_matches_too():
    _run(200, 72, 136, False, True, 2, True, use_tc=0)
    _run(200, 72, 136, True, False, 4, False, use_tc=0, scale=3.0)


def test_step_shape_forward_fc():
    # the depth-20 MLP up-projection shape with the relu^2 epilogue
    _run(4096, 5120, 1280, True, True, 2, True, seed=7)
