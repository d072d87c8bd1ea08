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


# Gradients (bf16 outputs of fp32 accumulations over bf16-rounded P and dS):
# relative RMS <= 1e-2 and max |err| <= 2e-2 of the reference's largest
# magnitude. P, dS and the outputs are each rounded to bf16 once (relative
# 2^-9 = 0.2 % per element), which puts the RMS error near 0.5 %. Both scales
# have a floor of 0.05: with unit-normal inputs the gradient entries are of
# order 0.1 to 10, and where the exact gradient vanishes (a window of 1: P = 1,
# D = dP, so dS = 0 and dQ = 0) what remains is rounding noise of order 1e-6.
GRAD_REL_RMS = 1e-2
GRAD_MAX_REL = 2e-2
GRAD_FLOOR = 0.05


def assert_grad_parity(g_gpu, g_ref, what=""):
    g_gpu, g_ref = to64(g_gpu), to64(g_ref)
    assert g_gpu.shape == g_ref.shape, (what, g_gpu.shape, g_ref.shape)
    assert np.isfinite(g_gpu).all(), f"{what}: non-finite gradient"
    scale = max(float(np.abs(g_ref).max()), GRAD_FLOOR)
    rms_ref = max(float(np.sqrt(np.mean(g_ref ** 2))), GRAD_FLOOR)
    max_abs = float(np.abs(g_gpu - g_ref).max())
    rms_err = float(np.sqrt(np.mean((g_gpu - g_ref) ** 2)))
    assert max_abs <= GRAD_MAX_REL * scale, f"{what}: max |err| {max_abs:.3e} > {GRAD_MAX_REL} x {scale:.3e}"
    assert rms_err <= GRAD_REL_RMS * rms_ref, f"{what}: RMS err {rms_err:.3e} > {GRAD_REL_RMS} x {rms_ref:.3e}"
    return {"max_abs": max_abs, "rel_rms": rms_err / rms_ref}
