"""Shared helpers of the GPU parity tests: upload seeded bit patterns, compare with the oracle."""
import numpy as np

import mfa_inputs as mi

# Tolerances on max |GPU - oracle| (outputs in the input type, LSE in fp32).
TOL_O = {mi.FP16: 4e-3, mi.BF16: 1.6e-2}
TOL_LSE = 1e-3


def to_torch(bits, dtype, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    t = t.view(torch.float16 if dtype == mi.FP16 else torch.bfloat16)
    return t.to(device)


def from_torch(t):
    """Exact fp64 copy of a CUDA fp16/bf16/fp32 tensor."""
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


def check_close(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    """Max-abs comparison; non-finite GPU values fail; -inf LSE must match exactly."""
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    err_o = float(np.max(np.abs(o_gpu - o_ref))) if o_ref.size else 0.0
    assert err_o <= TOL_O[dtype], f"{what}: max |O - oracle| = {err_o:.3e} > {TOL_O[dtype]:.1e}"
    if lse_gpu is not None:
        inf_ref = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), inf_ref), f"{what}: -inf LSE rows differ"
        fin = ~inf_ref
        assert np.all(np.isfinite(lse_gpu[fin])), f"{what}: non-finite LSE"
        err_l = float(np.max(np.abs(lse_gpu[fin] - lse_ref[fin]))) if fin.any() else 0.0
        assert err_l <= TOL_LSE, f"{what}: max |LSE - oracle| = {err_l:.3e} > {TOL_LSE:.1e}"
        return err_o, err_l
    return err_o, 0.0
