"""Shared helpers of the GPU tests: run the CUDA step through the C ABI on
seeded inputs, and compare with the float64 oracle."""
import numpy as np

import synth

# Tolerances of the two precisions: |loss - loss_ref| and per-tensor
# relative L2 error ||g - g_ref|| / ||g_ref|| of every gradient.
TOL = {"bf16": (2e-2, 3e-2), "fp32": (1e-4, 1e-3)}


def to_device_weights(bits, values, precision):
    import torch
    if precision == "bf16":
        return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(values).cuda()


def gpu_step(model, weights, tok, tgt, ws=None):
    """Runs nc_forward_backward; returns (loss, grads as numpy fp32)."""
    import torch
    B, T = tok.shape
    n = model.num_params()
    grads = torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")
    loss = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    if ws is None:
        ws = torch.empty(model.workspace_bytes(B, T), dtype=torch.uint8, device="cuda")
    model.forward_backward(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda(), weights, grads, loss, ws)
    code = model.check()
    assert code == 0, code
    return float(loss.item()), grads.cpu().numpy()


def compare(cfg, loss, grads, ref_loss, ref_grads, precision, tol=None):
    """Asserts the loss / per-tensor rel-L2 tolerances; returns the worst rel-L2."""
    tl, tg = tol or TOL[precision]
    assert np.isfinite(loss) and abs(loss - ref_loss) <= tl, (loss, ref_loss)
    worst = 0.0
    for name, r, c, off in synth.param_layout(cfg):
        g = grads[off:off + r * c].astype(np.float64)
        ref = ref_grads[off:off + r * c]
        assert np.all(np.isfinite(g)), name
        den = np.linalg.norm(ref)
        rel = np.linalg.norm(g - ref) / den if den > 0 else np.linalg.norm(g)
        worst = max(worst, rel)
        assert rel <= tg, (name, rel)
    return worst
