"""The failure path on a live GPU, without a fault: a bounded wait that nothing will satisfy.

With MFA_DEBUG_WITHHOLD_MMA the forward's MMA thread issues nothing, so the softmax warps' first
wait for S can never complete. Every mbarrier wait in the kernels polls %globaltimer and gives up
after 2 s: the kernel must then record MFA_ERR_DEVICE_TIMEOUT (with the wait's location) in the
device status word, write out = 0 and lse = -inf, release its TMEM and return; the CUDA context
stays usable and the next call computes normally."""
import time

import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu

MFA_ERR_DEVICE_TIMEOUT = -21


# (-1, -1): the two-Q-tile CTA shape; (64, 0): a sliding window, which runs one Q tile per CTA
@pytest.mark.parametrize("window", [(-1, -1), (64, 0)])
def test_wait_runs_out_reports_timeout_and_context_survives(cuda_device, window):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    case = mi.PrefillCase("one_cta", 1, 1, 1, 128, 128, 64, mi.FP16, True, seed=101)
    q, k, v = case.tensors()
    qt, kt, vt = (to_torch(x, case.dtype) for x in (q, k, v))
    mfa.mfa_device_status()  # clear
    old = mfa.mfa_debug_set_flags(mfa.MFA_DEBUG_WITHHOLD_MMA)
    try:
        t0 = time.time()
        out, lse = mfa.mfa_fwd(qt, kt, vt, scale=case.scale_f32(), causal=True, window=window)
        torch.cuda.synchronize()
        dt = time.time() - t0
    finally:
        mfa.mfa_debug_set_flags(old)
    code, where = mfa.mfa_device_status()
    assert code == MFA_ERR_DEVICE_TIMEOUT, (code, where)
    assert where in (1001, 1002), where          # a softmax warpgroup's wait for S
    assert 1.5 < dt < 60.0, dt
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    # the context is intact: the same call without the flag matches the oracle
    out, lse = mfa.mfa_fwd(qt, kt, vt, scale=case.scale_f32(), causal=True, window=window)
    torch.cuda.synchronize()
    w = lambda x: mi.widen(x, case.dtype)
    o_ref, l_ref = oracle.attention(w(q), w(k), w(v), case.scale_f32(), True, *window)
    check_close(from_torch(out), from_torch(lse), o_ref, l_ref, case.dtype, "after timeout")
    assert mfa.mfa_device_status() == (0, 0)
