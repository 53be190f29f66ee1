"""The allocation-free decode entry point (mfa_decode_splitkv_noalloc).

Callers such as serving engines that reserve all of HBM for their KV pool, or code running
inside an allocator callback, cannot allocate a decode workspace; this entry point uses a fixed
device array inside the library instead. Here it is called through the C ABI twice in a row (two
different shapes, so the second call reuses what the first left in the shared array) and each
result must match both the fp64 oracle's decode and the regular entry point's within the parity
tolerances. This file is collected last so that a failure here cannot hide the rest of the suite.
"""
import ctypes

import numpy as np
import pytest

import mfa_inputs as mi
import oracle
from gpu_util import TOL_LSE, TOL_O, check_close, from_torch, to_torch

pytestmark = pytest.mark.gpu


def _call_noalloc(mfa, case, qt, kt, vt, tt, lt, out, lse, stream):
    B, Hq, Nq, D = qt.shape
    return mfa.lib.mfa_decode_splitkv_noalloc(
        qt.data_ptr(), kt.data_ptr(), vt.data_ptr(), tt.data_ptr(), lt.data_ptr(), out.data_ptr(),
        lse.data_ptr(), B, Nq, Hq, kt.shape[2], D, 16, tt.shape[1], kt.shape[0],
        ctypes.c_float(case.scale_f32()), int(case.causal), ctypes.c_float(case.softcap),
        case.dtype, ctypes.c_void_p(stream.cuda_stream))


def test_noalloc_decode_matches_workspace_decode_twice_in_a_row(cuda_device):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    stream = torch.cuda.current_stream()
    cases = [mi.DecodeCase("noalloc_a", 4, 1, 32, 8, 128, mi.BF16, 100, 5000, seed=81),
             mi.DecodeCase("noalloc_b", 3, 4, 16, 4, 64, mi.FP16, 1, 900, seed=82)]
    for case in cases:
        q, k, v, table, lens = case.tensors()
        qt, kt, vt = (to_torch(x, case.dtype) for x in (q, k, v))
        tt = torch.from_numpy(table).cuda()
        lt = torch.from_numpy(lens).cuda()
        out = torch.empty_like(qt)
        lse = torch.empty(qt.shape[:3], dtype=torch.float32, device="cuda")
        rc = _call_noalloc(mfa, case, qt, kt, vt, tt, lt, out, lse, stream)
        assert rc == 0, mfa.mfa_status_string(rc)
        ref_o, ref_l = mfa.mfa_decode_splitkv(qt, kt, vt, tt, lt, scale=case.scale_f32(),
                                              causal=case.causal, softcap=case.softcap)
        torch.cuda.synchronize()
        o, l, ro, rl = from_torch(out), from_torch(lse), from_torch(ref_o), from_torch(ref_l)
        w = lambda x: mi.widen(x, case.dtype)
        oo, ol = oracle.decode(w(q), w(k), w(v), table, lens, case.scale_f32(), case.causal,
                               case.softcap)
        check_close(o, l, oo, ol, case.dtype, case.name + " vs oracle")
        assert np.all(np.isfinite(o))
        assert np.max(np.abs(o - ro)) <= TOL_O[case.dtype], case.name
        fin = np.isfinite(rl)
        assert np.array_equal(np.isneginf(l), np.isneginf(rl))
        assert np.max(np.abs(l[fin] - rl[fin])) <= TOL_LSE, case.name
    assert mfa.mfa_device_status() == (0, 0)


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    """A shape whose workspace exceeds the fixed array is refused before anything runs."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    need = mfa.mfa_decode_workspace_size(64, 4, 32, 8, 128, 65536)
    assert need > mfa.MFA_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(64, 32, 4, 128, dtype=torch.bfloat16, device="cuda")
    pages = torch.zeros(1, 16, 8, 128, dtype=torch.bfloat16, device="cuda")
    small = torch.zeros(64, 16, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty(64, 32, 4, dtype=torch.float32, device="cuda")
    rc = mfa.lib.mfa_decode_splitkv_noalloc(
        q.data_ptr(), pages.data_ptr(), pages.data_ptr(), small.data_ptr(), small.data_ptr(),
        out.data_ptr(), lse.data_ptr(), 64, 4, 32, 8, 128, 16, 65536, 1, ctypes.c_float(0.088), 1,
        ctypes.c_float(0.0), mi.BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -23, mfa.mfa_status_string(rc)
