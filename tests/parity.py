"""Tolerances for comparing the CUDA path with the fp64 oracle.

O (bf16 output, fp32 accumulation): max |err| <= 2e-2 and relative RMS
||O - O*||_2 / ||O*||_2 <= 1e-2 over the compared tensor; LSE (fp32):
max |err| <= 1e-3. Integer and index work (the paged gather) is bit-exact.
"""

import numpy as np
import torch

O_MAX_ABS = 2e-2
O_REL_RMS = 1e-2
LSE_MAX_ABS = 1e-3


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def assert_parity(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    o_gpu, o_ref = to64(o_gpu), to64(o_ref)
    assert o_gpu.shape == o_ref.shape, (what, o_gpu.shape, o_ref.shape)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    max_abs = float(err.max())
    rel = float(np.linalg.norm(o_gpu - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    assert max_abs <= O_MAX_ABS, f"{what}: max |err| {max_abs:.3e} > {O_MAX_ABS}"
    assert rel <= O_REL_RMS, f"{what}: relative RMS {rel:.3e} > {O_REL_RMS}"
    out = {"o_max_abs": max_abs, "o_rel_rms": rel}
    if lse_gpu is not None:
        lse_gpu, lse_ref = to64(lse_gpu), to64(lse_ref)
        assert np.isfinite(lse_gpu).all(), f"{what}: non-finite LSE"
        lmax = float(np.abs(lse_gpu - lse_ref).max())
        assert lmax <= LSE_MAX_ABS, f"{what}: LSE max |err| {lmax:.3e} > {LSE_MAX_ABS}"
        out["lse_max_abs"] = lmax
    return out
