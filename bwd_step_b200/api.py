"""Thin Python binding of the step's C ABI (argument marshalling only).

Every computation runs in the CUDA library; this module only turns torch
tensors (device memory allocated by PyTorch) into pointers and checks their
dtype, device and contiguity.
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import NcConfig, lib

PRECISIONS = {"bf16": _lib.NC_PREC_BF16, "fp32": _lib.NC_PREC_FP32_DEBUG}


class NcError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {lib().nc_status_string(code).decode()} ({code})")


def _ok(code: int, what: str):
    if code != _lib.NC_OK:
        raise NcError(code, what)


def _stream_handle(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ptr(t, dtype=None, name="tensor", on_device=True, device=None):
    """Pointer to a contiguous tensor of the given dtype, on the GPU (on_device)
    or in host memory: a host pointer handed to a kernel would fault the GPU.
    With `device` (a CUDA ordinal) a device tensor must live on that GPU: a
    buffer on another GPU would reach the kernels as peer memory."""
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if bool(t.is_cuda) != on_device:
        raise ValueError(f"{name} must be in {'device' if on_device else 'host'} memory")
    if on_device and device is not None and t.device.index != device:
        raise ValueError(f"{name} is on cuda:{t.device.index}, the model on cuda:{device}")
    return ctypes.c_void_p(t.data_ptr())


def _check_extents(n_params, vocab, tokens, targets=None, weights=None, grads=None, loss=None, logits=None):
    """The C ABI takes bare pointers, so sizes are checked here: a buffer shorter
    than the flat layout (or than [B, T, V] logits) would be written past its end."""
    if tokens.dim() != 2:
        raise ValueError("tokens must be [B, T]")
    if targets is not None and tuple(targets.shape) != tuple(tokens.shape):
        raise ValueError("targets must have the shape of tokens")
    for name, t, need in (("weights", weights, n_params), ("grads", grads, n_params), ("loss", loss, 1),
                          ("logits", logits, tokens.numel() * vocab)):
        if t is not None and t.numel() < need:
            raise ValueError(f"{name} holds {t.numel()} elements, needs {need}")


def adamw_step(groups, step, master, weights, grads, m, v, stream=None):
    """AdamW update of parameter groups [(offset, count, lr, beta1, beta2, eps,
    weight_decay)] of the flat fp32 master weights (in place), the moments m and
    v (in place) and the compute copy `weights` (bf16 or fp32); step >= 1."""
    import torch
    n = master.numel()
    for name, t in (("weights", weights), ("grads", grads), ("m", m), ("v", v)):
        if t.numel() != n:
            raise ValueError(f"{name} holds {t.numel()} elements, master {n}")
    dev = master.device.index
    arr = (_lib.NcAdamwGroup * max(len(groups), 1))(
        *[_lib.NcAdamwGroup(int(o), int(c), float(lr), float(b1), float(b2), float(e), float(wd))
          for o, c, lr, b1, b2, e, wd in groups])
    if weights.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("weights must be bf16 or fp32")
    _ok(lib().nc_adamw_step(arr, len(groups), n, int(step), _ptr(master, torch.float32, "master", device=dev),
                            _ptr(weights, None, "weights", device=dev), 1 if weights.dtype == torch.bfloat16 else 0,
                            _ptr(grads, torch.float32, "grads", device=dev), _ptr(m, torch.float32, "m", device=dev),
                            _ptr(v, torch.float32, "v", device=dev), ctypes.c_void_p(_stream_handle(stream))),
        "nc_adamw_step")


def launch_count() -> int:
    """Kernels launched by the CUDA library in this process so far."""
    return int(lib().nc_launch_count())


class Model:
    """A model handle: shape, precision and the flat parameter layout."""

    def __init__(self, cfg, precision: str = "bf16"):
        get = (lambda k: cfg[k]) if isinstance(cfg, dict) else (lambda k: getattr(cfg, k))
        self.cfg = NcConfig(get("vocab"), get("d_model"), get("n_layer"), get("n_head"), get("n_kv_head"),
                            get("head_dim"), get("mlp_mult"), float(get("softcap")), float(get("rope_base")))
        self.precision = precision
        h = ctypes.c_void_p()
        _ok(lib().nc_model_create(ctypes.byref(self.cfg), PRECISIONS[precision], ctypes.byref(h)),
            "nc_model_create")
        self._h = h
        import torch
        # nc_model_create bound the model to the current device; every device
        # tensor handed to it later must live there
        self.device = torch.cuda.current_device()

    def close(self):
        if getattr(self, "_h", None):
            lib().nc_model_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def weight_dtype(self):
        import torch
        return torch.bfloat16 if self.precision == "bf16" else torch.float32

    def num_params(self) -> int:
        return int(lib().nc_num_params(self._h))

    def layout(self):
        out = []
        i = 0
        name, off = ctypes.c_char_p(), ctypes.c_int64()
        r, c = ctypes.c_int(), ctypes.c_int()
        while lib().nc_param_layout(self._h, i, ctypes.byref(name), ctypes.byref(off), ctypes.byref(r),
                                    ctypes.byref(c)) == _lib.NC_OK:
            out.append((name.value.decode(), r.value, c.value, off.value))
            i += 1
        return out

    def workspace_bytes(self, B: int, T: int) -> int:
        return int(lib().nc_workspace_bytes(self._h, B, T))

    def _dev(self, t, dtype, name):
        """Pointer to a device tensor on the model's GPU."""
        return _ptr(t, dtype, name, device=self.device)

    def forward_backward(self, tokens, targets, weights, grads, loss, workspace, stream=None):
        """One step on device tensors; grads (fp32) and loss (fp32 [1]) are overwritten."""
        import torch
        _check_extents(self.num_params(), self.cfg.vocab, tokens, targets, weights, grads, loss)
        B, T = tokens.shape
        _ok(lib().nc_forward_backward(self._h, self._dev(tokens, torch.int32, "tokens"),
                                      self._dev(targets, torch.int32, "targets"), B, T,
                                      self._dev(weights, self.weight_dtype, "weights"),
                                      self._dev(grads, torch.float32, "grads"),
                                      self._dev(loss, torch.float32, "loss"),
                                      self._dev(workspace, None, "workspace"),
                                      workspace.numel() * workspace.element_size(),
                                      ctypes.c_void_p(_stream_handle(stream))), "nc_forward_backward")

    def forward_backward_host(self, h_tokens, h_targets, weights, grads, workspace, stream=None) -> float:
        """One step with host (ideally pinned) int32 token/target tensors; returns the loss."""
        import torch
        _check_extents(self.num_params(), self.cfg.vocab, h_tokens, h_targets, weights, grads)
        B, T = h_tokens.shape
        out = ctypes.c_float()
        _ok(lib().nc_forward_backward_host(self._h, _ptr(h_tokens, torch.int32, "tokens", on_device=False),
                                           _ptr(h_targets, torch.int32, "targets", on_device=False), B, T,
                                           self._dev(weights, self.weight_dtype, "weights"),
                                           self._dev(grads, torch.float32, "grads"), ctypes.byref(out),
                                           self._dev(workspace, None, "workspace"),
                                           workspace.numel() * workspace.element_size(),
                                           ctypes.c_void_p(_stream_handle(stream))), "nc_forward_backward_host")
        return out.value

    def forward_logits(self, tokens, weights, logits, workspace, stream=None):
        """Softcapped logits [B, T, V] of the forward pass (weight dtype)."""
        import torch
        _check_extents(self.num_params(), self.cfg.vocab, tokens, weights=weights, logits=logits)
        B, T = tokens.shape
        _ok(lib().nc_forward_logits(self._h, self._dev(tokens, torch.int32, "tokens"), B, T,
                                    self._dev(weights, self.weight_dtype, "weights"),
                                    self._dev(logits, self.weight_dtype, "logits"),
                                    self._dev(workspace, None, "workspace"),
                                    workspace.numel() * workspace.element_size(),
                                    ctypes.c_void_p(_stream_handle(stream))), "nc_forward_logits")

    def kv_cache_bytes(self, B: int, T_max: int) -> int:
        return int(lib().nc_kv_cache_bytes(self._h, B, T_max))

    def inference_workspace_bytes(self, B: int, T_max: int) -> int:
        return int(lib().nc_inference_workspace_bytes(self._h, B, T_max))

    def prefill(self, tokens, weights, kv_cache, T_max, logits, workspace, stream=None):
        """Forward over the prompt tokens [B, T] (device int32); fills cache
        positions 0..T-1 and writes the last position's softcapped logits [B, V]."""
        import torch
        B, T = tokens.shape
        self._check_inference(B, T_max, weights, kv_cache, logits)
        _ok(lib().nc_prefill(self._h, self._dev(tokens, torch.int32, "tokens"), B, T,
                             self._dev(weights, self.weight_dtype, "weights"), self._dev(kv_cache, None, "kv_cache"),
                             int(T_max), self._dev(logits, self.weight_dtype, "logits"),
                             self._dev(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
                             ctypes.c_void_p(_stream_handle(stream))), "nc_prefill")

    def decode_step(self, tokens, pos, weights, kv_cache, T_max, logits, workspace, stream=None):
        """One new token per row (device int32 [B]) at position pos: appends to
        the cache and writes that position's softcapped logits [B, V]."""
        import torch
        B = tokens.shape[0]
        if tokens.dim() != 1:
            raise ValueError("tokens must be [B]")
        self._check_inference(B, T_max, weights, kv_cache, logits)
        _ok(lib().nc_decode_step(self._h, self._dev(tokens, torch.int32, "tokens"), B, int(pos),
                                 self._dev(weights, self.weight_dtype, "weights"),
                                 self._dev(kv_cache, None, "kv_cache"), int(T_max),
                                 self._dev(logits, self.weight_dtype, "logits"),
                                 self._dev(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
                                 ctypes.c_void_p(_stream_handle(stream))), "nc_decode_step")

    def _check_inference(self, B, T_max, weights, kv_cache, logits):
        if weights.numel() < self.num_params():
            raise ValueError("weights shorter than the flat layout")
        if kv_cache.numel() * kv_cache.element_size() < self.kv_cache_bytes(B, T_max):
            raise ValueError("kv_cache smaller than kv_cache_bytes(B, T_max)")
        if logits.numel() < B * self.cfg.vocab:
            raise ValueError("logits must hold [B, V]")

    def set_recompute(self, mlp: bool):
        """Recompute the MLP's relu(u), relu(u)^2 in the backward instead of
        saving them per layer (less workspace; query workspace_bytes afterwards)."""
        _ok(lib().nc_set_recompute(self._h, _lib.NC_RECOMPUTE_MLP if mlp else _lib.NC_RECOMPUTE_NONE),
            "nc_set_recompute")

    def set_lm_head(self, mode: str = "fused", chunk_rows: int = 0):
        """LM head strategy: "fused" (logits never stored; bf16 only) or
        "materialised" (logit chunks plus a cross-entropy pass); chunk_rows 0 =
        default.  Query workspace_bytes afterwards: it depends on both."""
        code = {"fused": _lib.NC_LM_HEAD_FUSED, "materialised": _lib.NC_LM_HEAD_MATERIALISED}[mode]
        _ok(lib().nc_set_lm_head(self._h, code, int(chunk_rows)), "nc_set_lm_head")

    def check(self, stream=None) -> int:
        """Synchronise the stream and return (and clear) the device status code."""
        return int(lib().nc_check(self._h, ctypes.c_void_p(_stream_handle(stream))))

    def profile(self, enable: bool):
        """Start (clearing) or stop per-kernel-class event timing."""
        _ok(lib().nc_profile_enable(self._h, 1 if enable else 0), "nc_profile_enable")

    def profile_read(self, stream=None):
        """Aggregated rows {kernel, launches, ms, flops, bytes} (synchronises the stream)."""
        rows = (_lib.NcProfileRow * 32)()
        n = lib().nc_profile_read(self._h, ctypes.c_void_p(_stream_handle(stream)), rows, 32)
        if n < 0:
            raise NcError(n, "nc_profile_read")
        return [dict(kernel=r.kernel.decode(), launches=r.launches, ms=r.ms, flops=r.flops, bytes=r.bytes)
                for r in rows[:n]]

    def grad_buckets(self):
        """[(offset, count)] of the flat gradient buffer in the order the backward
        finishes them: LM head, layers last to first, token embedding."""
        n = lib().nc_grad_bucket_count(self._h)
        if n < 0:
            raise NcError(n, "nc_grad_bucket_count")
        out = []
        for i in range(n):
            off, cnt = ctypes.c_int64(), ctypes.c_int64()
            _ok(lib().nc_grad_bucket(self._h, i, ctypes.byref(off), ctypes.byref(cnt)), "nc_grad_bucket")
            out.append((off.value, cnt.value))
        return out

    def set_grad_events(self, events):
        """Have every step record events[i] (torch.cuda.Event, already created by a
        record) when gradient bucket i is final; an empty list clears them."""
        handles = (ctypes.c_void_p * max(len(events), 1))(*[ctypes.c_void_p(e.cuda_event) for e in events])
        _ok(lib().nc_set_grad_events(self._h, handles, len(events)), "nc_set_grad_events")
        self._grad_events = list(events)  # the handles must outlive their use

    def debug_expired_wait(self, max_iters: int, stream=None):
        _ok(lib().nc_debug_expired_wait(self._h, max_iters, ctypes.c_void_p(_stream_handle(stream))),
            "nc_debug_expired_wait")
