"""Helpers of the GPU parity tests (device copies, tolerance checks)."""
import numpy as np
import torch

ATTN_MAX_ABS = 2e-3     # max |gpu - fp64 oracle| over an output tensor
ATTN_REL_L2 = 1e-3      # ||gpu - oracle||_2 / ||oracle||_2 over an output tensor


def dev(a, dtype=None):
    """NumPy -> CUDA tensor (bf16 bit patterns stay uint16 -> bfloat16 view)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(a).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def check_attention(out_gpu, out_ref, lse_gpu=None, lse_ref=None, what=""):
    o = np.asarray(out_gpu, np.float64)
    r = np.asarray(out_ref, np.float64)
    err = np.abs(o - r)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(o - r) / max(np.linalg.norm(r), 1e-30))
    assert max_abs <= ATTN_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {ATTN_MAX_ABS}"
    assert rel <= ATTN_REL_L2, f"{what}: rel-L2 {rel:.3e} > {ATTN_REL_L2}"
    if lse_gpu is not None:
        lg, lr = np.asarray(lse_gpu, np.float64), np.asarray(lse_ref, np.float64)
        fin = np.isfinite(lr)
        assert np.array_equal(np.isfinite(lg), fin), f"{what}: lse finiteness differs"
        assert np.all(np.abs(lg[fin] - lr[fin]) <= 1e-4 * np.maximum(1, np.abs(lr[fin]))), f"{what}: lse"
    return max_abs, rel
