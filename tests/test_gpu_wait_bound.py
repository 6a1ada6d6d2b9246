"""The bounded pipeline waits of the scoring kernels.

Every mbarrier wait of the scoring kernels gives up after a bound, records
KVC_DEV_ERR_TIMEOUT in the device error word, lets the copies and MMAs it
already issued land, frees its TMEM and returns.  The test library
``libkvc_shortwait.so`` is the same scoring code built with a bound of a few
nanoseconds, so its first wait that does not succeed at once gives up: the
call must still return, the error bit must be set, and the CUDA context must
stay usable -- a regular call right after it gives the oracle's scores.  No
wait is made to hang and nothing faults: the short bound only ends waits that
would otherwise have completed.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import long_context_kv_window_b200 as kvc
import oracle
import workloads
from long_context_kv_window_b200 import build as kbuild
from tests import parity
from tests.gpu_helpers import dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def short_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvc.lib()
    torch.cuda.set_device(0)
    if not os.path.exists(kbuild.SHORTWAIT_LIB):
        raise FileNotFoundError(f"{kbuild.SHORTWAIT_LIB} is missing: run `python -m long_context_kv_window_b200.build`")
    L = ctypes.CDLL(kbuild.SHORTWAIT_LIB)
    for name in ("kvc_score", "kvc_score_workspace_size", "kvc_last_error"):
        args, res = kvc._SIGS[name]
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


def test_wait_bound_reports_timeout_and_the_context_stays_usable(short_lib):
    cfg = workloads.shrink(workloads.C2, N=4096, k_kv=256, n_hitters=8, seed=77)
    lay = workloads.make_layer(cfg)
    q, k = dev_bf16(lay.q), dev_bf16(lay.k)
    p = kvc.score_params(cfg.H, cfg.Hkv, cfg.d, cfg.w)
    ws = torch.empty(kvc.score_workspace_size(p, 1, cfg.N), dtype=torch.uint8, device="cuda")
    scores = torch.zeros((cfg.Hkv, cfg.N), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream()
    for call in range(2):
        err.zero_()
        rc = short_lib.kvc_score(ctypes.c_void_p(q.data_ptr()), q.stride(0), q.stride(1),
                                 ctypes.c_void_p(k.data_ptr()), k.stride(0), k.stride(1), cfg.N, ctypes.byref(p),
                                 ctypes.c_void_p(scores.data_ptr()), None, None, ctypes.c_void_p(ws.data_ptr()),
                                 ws.numel(), ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(st.cuda_stream))
        assert rc == kvc.KVC_OK, short_lib.kvc_last_error().decode()
        torch.cuda.synchronize()  # the call returned and its kernels finished
        assert err.item() & kvc.KVC_DEV_ERR_TIMEOUT, f"call {call}: no wait gave up (error word {err.item()})"

    # the regular library in the same context afterwards
    err.zero_()
    good = kvc.kvc_score(q, k, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.get().window_scores(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale)
    parity.assert_scores_close(good.cpu().numpy(), ref, what="scores after the short-wait calls")
    assert np.isfinite(good.cpu().numpy()).all()
