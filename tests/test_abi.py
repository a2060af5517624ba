"""CPU-side checks of the C ABI: the in-tree library loads, exports every
entry point the public header declares, and refuses to run without a GPU."""
import ctypes
import glob
import os
import re

import pytest

import bwd_step_b200
from bwd_step_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(nc_\w+)\s*\(", text))
    return names


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("nc_model_create", "nc_forward_backward", "nc_forward_logits", "nc_workspace_bytes",
              "nc_param_layout", "nc_check"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = bwd_step_b200.lib()
    for n in sorted(_declared()):
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"


def test_status_strings():
    L = bwd_step_b200.lib()
    for code in range(-7, 1):
        assert L.nc_status_string(code)
    assert L.nc_status_string(0) == b"ok"


def test_create_rejects_bad_config_without_touching_a_device():
    cfg = _lib.NcConfig(512, 64, 2, 4, 1, 16, 4, 15.0, 10000.0)
    out = ctypes.c_void_p()
    L = bwd_step_b200.lib()
    assert L.nc_model_create(None, 0, ctypes.byref(out)) == _lib.NC_ERR_INVALID_ARG
    assert L.nc_model_create(ctypes.byref(cfg), 7, ctypes.byref(out)) == _lib.NC_ERR_INVALID_ARG
    bad = _lib.NcConfig(512, 64, 2, 4, 1, 24, 4, 15.0, 10000.0)  # head_dim 24
    assert L.nc_model_create(ctypes.byref(bad), 0, ctypes.byref(out)) == _lib.NC_ERR_UNSUPPORTED_SHAPE
    bad = _lib.NcConfig(512, 64, 2, 3, 2, 16, 4, 15.0, 10000.0)  # n_head % n_kv_head
    assert L.nc_model_create(ctypes.byref(bad), 0, ctypes.byref(out)) == _lib.NC_ERR_UNSUPPORTED_SHAPE
    bad = _lib.NcConfig(512, 64, 2, 4, 1, 16, 4, -1.0, 10000.0)  # softcap <= 0
    assert L.nc_model_create(ctypes.byref(bad), 0, ctypes.byref(out)) == _lib.NC_ERR_INVALID_ARG
    assert out.value is None


def test_no_cpu_fallback():
    """Without a CUDA device the product path refuses to run."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(bwd_step_b200.NcError) as e:
        bwd_step_b200.Model({"vocab": 512, "d_model": 64, "n_layer": 2, "n_head": 4, "n_kv_head": 1,
                             "head_dim": 16, "mlp_mult": 4, "softcap": 15.0, "rope_base": 10000.0})
    assert e.value.code == _lib.NC_ERR_NO_DEVICE


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "bwd_step_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.*"), recursive=True):
        if path.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
            src = open(path).read()
            assert not re.search(r"\boracle\b", src), path


def test_marshalling_rejects_memory_on_the_wrong_side():
    """A host pointer handed to a kernel would fault the GPU: the binding checks
    where every tensor lives before passing its address."""
    import torch
    from bwd_step_b200.api import _ptr
    t = torch.zeros(8, dtype=torch.int32)
    with pytest.raises(ValueError):
        _ptr(t, torch.int32, "tokens")  # device memory expected
    assert _ptr(t, torch.int32, "tokens", on_device=False).value == t.data_ptr()
    with pytest.raises(TypeError):
        _ptr(t, torch.float32, "grads", on_device=False)
    with pytest.raises(ValueError):
        _ptr(torch.zeros(4, 4, dtype=torch.int32).t(), torch.int32, "tokens", on_device=False)


def test_marshalling_rejects_a_tensor_on_another_gpu():
    """A buffer on another GPU would reach the model's kernels as peer memory:
    the binding compares every device tensor's ordinal with the model's."""
    import torch
    from bwd_step_b200.api import _ptr

    class OnGpu:  # stands in for a CUDA tensor (no GPU is needed for the check)
        dtype = torch.float32
        is_cuda = True

        def __init__(self, index):
            self.device = torch.device("cuda", index)

        def is_contiguous(self):
            return True

        def data_ptr(self):
            return 4096

    assert _ptr(OnGpu(0), torch.float32, "grads", device=0).value == 4096
    with pytest.raises(ValueError, match="cuda:1"):
        _ptr(OnGpu(1), torch.float32, "grads", device=0)


def test_marshalling_checks_buffer_extents():
    """Buffers shorter than the flat layout or the logits are refused before any
    pointer reaches the library."""
    import torch
    from bwd_step_b200.api import _check_extents
    tok = torch.zeros(2, 8, dtype=torch.int32)
    w, g, l = torch.zeros(100), torch.zeros(100), torch.zeros(1)
    _check_extents(100, 16, tok, tok.clone(), w, g, l)
    for bad in (dict(targets=torch.zeros(2, 7, dtype=torch.int32)), dict(weights=torch.zeros(99)),
                dict(grads=torch.zeros(99)), dict(loss=torch.zeros(0))):
        args = dict(targets=tok.clone(), weights=w, grads=g, loss=l)
        args.update(bad)
        with pytest.raises(ValueError):
            _check_extents(100, 16, tok, **args)
    _check_extents(100, 16, tok, weights=w, logits=torch.zeros(2 * 8 * 16))
    with pytest.raises(ValueError):
        _check_extents(100, 16, tok, weights=w, logits=torch.zeros(2 * 8 * 16 - 1))
    with pytest.raises(ValueError):
        _check_extents(100, 16, torch.zeros(16, dtype=torch.int32), weights=w)
