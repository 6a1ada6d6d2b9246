"""kvc_score_noalloc: window scoring for callers that cannot allocate.

Callers such as an operator inside another runtime's plugin interface (no
scratch buffer offered) or a serving loop that must not call cudaMalloc once
running (it can synchronise the device) use this entry point; its scratch is
a static device array inside libkvc instead of a caller workspace.  It must
give the same scores as kvc_score -- checked here on two calls in a row with
different inputs, since the static scratch keeps the previous call's
contents -- and must reject sizes beyond its scratch without launching.

This file is collected last on purpose (its name) and is independent of the
other tests, so it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import long_context_kv_window_b200 as kvc
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvc.lib()
    torch.cuda.set_device(0)


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    for seed, with_tsp in ((71, False), (72, True)):
        cfg = workloads.shrink(workloads.C2, N=20000, n_hitters=16, seed=seed)
        lay = workloads.make_layer(cfg, with_x=False)
        q = workloads.torch_bf16(lay.q, "cuda")
        k = workloads.torch_bf16(lay.k, "cuda")
        tsp_ref = torch.empty(cfg.N, dtype=torch.float32, device="cuda") if with_tsp else None
        ref = kvc.kvc_score(q, k, tsp=tsp_ref)
        got = torch.full_like(ref, float("nan"))
        tsp_got = torch.full((cfg.N,), float("nan"), device="cuda") if with_tsp else None
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        kvc.kvc_score_noalloc(q, k, scores=got, tsp=tsp_got, dev_err=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        parity.assert_scores_close(got.cpu().numpy(), ref.cpu().numpy(), what=f"noalloc seed {seed}")
        if with_tsp:
            parity.assert_scores_close(tsp_got.cpu().numpy(), tsp_ref.cpu().numpy(), what="noalloc tsp")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = kvc.lib()
    p = kvc.score_params(32, 8, 128, 32)
    dummy = ctypes.c_void_p(256)  # never dereferenced: the size check fails first
    before = kvc.launch_count()
    rc = L.kvc_score_noalloc(dummy, 4096, 128, dummy, 1024, 128, 1 << 30, ctypes.byref(p), dummy, None, None,
                             None, None)
    assert rc == 4  # KVC_ERR_WORKSPACE
    assert "static scratch holds" in kvc.last_error()
    assert kvc.launch_count() == before
