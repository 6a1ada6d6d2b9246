"""Host-side argument checks of the Python binding.

The C entry points take raw pointers and cannot see how large a tensor is;
the binding checks every buffer against the sizes it passes (shape, dtype,
device, density) before anything reaches the library.  These tests run on
the CPU: the helpers are exercised directly, and the public wrappers with
their CUDA-only steps (the bf16 input check's device test, the device guard,
the stream lookup, the library itself) replaced by stand-ins that record the
call instead of launching anything.
"""
import ctypes

import pytest
import torch

import long_context_kv_window_b200 as kvc

CPU = torch.device("cpu")
f32, i32, bf = torch.float32, torch.int32, torch.bfloat16


# --------------------------------------------------------------------------- #
# helpers
# --------------------------------------------------------------------------- #
def test_dense_requires_exact_shape_dtype_and_contiguity():
    t = torch.empty((3, 5), dtype=f32)
    assert kvc._dense(t, "t", (3, 5), f32, CPU) is t
    with pytest.raises(ValueError):
        kvc._dense(t, "t", (3, 4), f32, CPU)
    with pytest.raises(ValueError):
        kvc._dense(torch.empty((5, 3), dtype=f32).t(), "t", (3, 5), f32, CPU)  # right shape, not dense
    with pytest.raises(TypeError):
        kvc._dense(t, "t", (3, 5), torch.float64, CPU)
    with pytest.raises(TypeError):
        kvc._dense(torch.empty((3, 5), dtype=f32, device="meta"), "t", (3, 5), f32, CPU)
    for dt in (bf, torch.int16, torch.uint16):
        kvc._dense(torch.empty((2, 2), dtype=dt), "t", (2, 2), kvc._BF16_BITS, CPU)
    with pytest.raises(TypeError):
        kvc._dense(torch.empty((2, 2), dtype=f32), "t", (2, 2), kvc._BF16_BITS, CPU)


def test_vector_counts_elements_of_any_shape():
    assert kvc._vector(None, "v", 7, f32, CPU) is None
    kvc._vector(torch.empty(7, dtype=f32), "v", 7, f32, CPU)
    kvc._vector(torch.empty((1, 7), dtype=f32), "v", 7, f32, CPU)
    with pytest.raises(ValueError):
        kvc._vector(torch.empty(8, dtype=f32), "v", 7, f32, CPU)
    with pytest.raises(ValueError):
        kvc._vector(torch.empty(14, dtype=f32)[::2], "v", 7, f32, CPU)
    with pytest.raises(TypeError):
        kvc._vector(torch.empty(7, dtype=torch.int64), "v", 7, i32, CPU)


def test_rows_accepts_row_strided_views_only_with_unit_columns():
    wide = torch.empty((4, 10), dtype=f32)
    kvc._rows(wide[:, :6], "m", 4, 6, f32, CPU)  # row stride 10, 6 columns used
    kvc._rows(wide, "m", 4, 6, f32, CPU)          # more columns than needed
    with pytest.raises(ValueError):
        kvc._rows(wide, "m", 3, 6, f32, CPU)
    with pytest.raises(ValueError):
        kvc._rows(wide[:, :5], "m", 4, 6, f32, CPU)
    with pytest.raises(ValueError):
        kvc._rows(torch.empty((10, 4), dtype=f32).t(), "m", 4, 6, f32, CPU)  # column stride 4
    with pytest.raises(ValueError):
        kvc._rows(torch.empty(40, dtype=f32), "m", 4, 6, f32, CPU)


def test_error_word_and_row_groups():
    kvc._err_word(None, CPU)
    kvc._err_word(torch.zeros(1, dtype=i32), CPU)
    with pytest.raises(TypeError):
        kvc._err_word(torch.zeros(1, dtype=torch.int64), CPU)
    with pytest.raises(TypeError):
        kvc._err_word(torch.zeros(0, dtype=i32), CPU)
    assert kvc._out_rows(8, 4) == 2
    for rows, grp in ((8, 3), (8, 0)):
        with pytest.raises(ValueError):
            kvc._out_rows(rows, grp)


# --------------------------------------------------------------------------- #
# wrappers, with the CUDA-only steps stubbed
# --------------------------------------------------------------------------- #
class _Lib:
    """Stands in for libkvc: records entry-point calls, returns KVC_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return kvc.KVC_OK
        return fn


@pytest.fixture
def lib(monkeypatch):
    fake = _Lib()
    real_bf16 = kvc._bf16

    def bf16_any_device(t, name, dim):
        if t.dtype not in kvc._BF16_BITS:
            return real_bf16(t, name, dim)  # raises the dtype error
        if t.dim() != dim:
            raise ValueError(f"{name} must have {dim} dimensions")
        if t.stride(-1) != 1:
            raise ValueError(f"{name} must be contiguous in its last dimension")
        return t

    monkeypatch.setattr(kvc, "lib", lambda: fake)
    monkeypatch.setattr(kvc, "_bf16", bf16_any_device)
    monkeypatch.setattr(kvc, "_call", lambda dev, fn, *args: fn(*args))
    monkeypatch.setattr(kvc, "_stream", lambda stream, dev: ctypes.c_void_p(0))
    return fake


def _ws():
    return torch.empty(16, dtype=torch.uint8)


def test_score_checks_outputs(lib):
    w, H, Hkv, d, n = 4, 8, 2, 64, 100
    q, k = torch.empty((w, H, d), dtype=bf), torch.empty((n, Hkv, d), dtype=bf)
    ok = dict(scores=torch.empty((Hkv, n), dtype=f32), tsp=torch.empty((1, n), dtype=f32),
              accum=torch.empty((Hkv, n), dtype=f32), ws=_ws(), dev_err=torch.zeros(1, dtype=i32))
    kvc.kvc_score(q, k, **ok)
    kvc.kvc_score_noalloc(q, k, **{a: b for a, b in ok.items() if a != "ws"})
    assert lib.calls == ["kvc_score", "kvc_score_noalloc"]
    bad = [dict(scores=torch.empty((Hkv, n + 1), dtype=f32)), dict(scores=torch.empty((Hkv, n), dtype=torch.float64)),
           dict(tsp=torch.empty(n - 1, dtype=f32)), dict(accum=torch.empty((Hkv + 1, n), dtype=f32)),
           dict(accum=torch.empty((n, Hkv), dtype=f32).t()), dict(dev_err=torch.zeros(1, dtype=torch.int64)),
           dict(ws=torch.empty(32, dtype=torch.uint8)[::2])]
    for b in bad:
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_score(q, k, **{**ok, **b})
    with pytest.raises(ValueError):
        kvc.kvc_score(q, torch.empty((n, Hkv, d), dtype=bf, device="meta"), **ok)  # inputs on two devices
    with pytest.raises(ValueError):
        kvc.kvc_score(q, torch.empty((n, Hkv, 128), dtype=bf), **ok)  # head_dim differs
    with pytest.raises(ValueError):
        kvc.kvc_score(q.view(1, w, H, d), k, **ok)  # varlen-shaped window
    assert lib.calls == ["kvc_score", "kvc_score_noalloc"]


def test_score_lse_checks_the_normalisers(lib):
    w, H, Hkv, d, n = 4, 8, 2, 64, 100
    q, k = torch.empty((w, H, d), dtype=bf), torch.empty((n, Hkv, d), dtype=bf)
    full = torch.empty((H, n), dtype=f32)          # a prefill attention's [H][n] log-sum-exp
    kvc.kvc_score_lse(q, k, full[:, n - w:].t(), ws=_ws())
    assert lib.calls == ["kvc_score_lse"]
    for bad in (full[:, n - w:], torch.empty((w, H), dtype=torch.float64), torch.empty((w, H + 1), dtype=f32),
                torch.empty((w, H), dtype=f32, device="meta")):
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_score_lse(q, k, bad, ws=_ws())
    with pytest.raises(ValueError):
        kvc.kvc_score_lse(q, k, full[:, n - w:].t(), scores=torch.empty((Hkv, n - 1), dtype=f32), ws=_ws())
    assert lib.calls == ["kvc_score_lse"]


def test_score_varlen_checks_seqlens_and_outputs(lib):
    B, w, H, Hkv, d, total = 3, 4, 8, 2, 64, 300
    q, k = torch.empty((B, w, H, d), dtype=bf), torch.empty((total, Hkv, d), dtype=bf)
    cu = torch.tensor([0, 100, 200, 300], dtype=i32)
    kvc.kvc_score_varlen(q, k, cu, 100, ws=_ws())
    for b in (dict(cu_seqlens=cu[:3]), dict(cu_seqlens=cu.long()),
              dict(scores=torch.empty((Hkv, total - 1), dtype=f32))):
        args = dict(cu_seqlens=cu, ws=_ws())
        args.update(b)
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_score_varlen(q, k, max_seqlen=100, **args)
    assert lib.calls == ["kvc_score_varlen"]


def test_select_checks_rows_budget_and_outputs(lib):
    rows, n, w, k = 8, 500, 16, 64
    S = torch.empty((rows, n + 12), dtype=f32)[:, :n]  # row-strided view
    idx = kvc.kvc_select_topk(S, w, 3, k, ws=_ws())
    assert tuple(idx.shape) == (rows, k)
    kvc.kvc_select_topk(S, w, 3, k, row_group=4, idx=torch.empty((2, k + 5), dtype=i32), ws=_ws())
    kvc.kvc_select_topk(S, w, 3, k, pooled=torch.empty((rows, n - w), dtype=f32))
    assert lib.calls == ["kvc_select_topk"] * 3
    bad = [dict(row_group=3), dict(n=n + 1), dict(idx=torch.empty((rows, k - 1), dtype=i32)),
           dict(idx=torch.empty((rows + 1, k), dtype=i32)), dict(idx=torch.empty((rows, k), dtype=torch.int64)),
           dict(pooled=torch.empty((rows, n), dtype=f32))]
    for b in bad:
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_select_topk(S, w, 3, k, ws=_ws(), **b)
    with pytest.raises(ValueError):
        kvc.kvc_select_topk(torch.empty(n, dtype=f32), w, 3, k, ws=_ws())  # one row must still be [1][n]
    assert lib.calls == ["kvc_select_topk"] * 3


def test_select_varlen_checks(lib):
    rows, total, w, k = 4, 900, 16, 50
    S = torch.empty((rows, total), dtype=f32)
    cu = torch.tensor([0, 300, 900], dtype=i32)
    idx, counts = kvc.kvc_select_topk_varlen(S, cu, 600, w, 1, k, row_group=2, ws=_ws())
    assert tuple(idx.shape) == (2, 2, k) and tuple(counts.shape) == (2,)
    for b in (dict(idx=torch.empty((2, 4, k), dtype=i32)), dict(counts=torch.empty(3, dtype=i32)),
              dict(row_group=3), dict(dev_err=torch.zeros(1, dtype=f32))):
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_select_topk_varlen(S, cu, 600, w, 1, k, ws=_ws(), **{"row_group": 2, **b})
    assert lib.calls == ["kvc_select_topk_varlen"]


def test_gather_kv_checks(lib):
    n, Hkv, d, kk = 200, 3, 64, 40
    k, v = torch.empty((n, Hkv, d), dtype=bf), torch.empty((n, Hkv, d), dtype=bf)
    ko, vo = kvc.kvc_gather_kv(k, v, torch.empty((Hkv, kk), dtype=i32))
    assert tuple(ko.shape) == (Hkv, kk, d) and tuple(vo.shape) == (Hkv, kk, d)
    kvc.kvc_gather_kv(k, None, torch.empty((1, kk), dtype=i32), k_out=torch.empty((Hkv, kk, d), dtype=torch.int16))
    assert lib.calls == ["kvc_gather_kv"] * 2
    idx = torch.empty((Hkv, kk), dtype=i32)
    bad = [dict(idx=torch.empty((2, kk), dtype=i32)), dict(idx=torch.empty(kk, dtype=i32)),
           dict(k_out=torch.empty((Hkv, kk + 1, d), dtype=bf)), dict(k_out=torch.empty((Hkv, kk, d), dtype=f32)),
           dict(v=torch.empty((n + 1, Hkv, d), dtype=bf)), dict(v_out=torch.empty((Hkv, kk, d + 8), dtype=bf))]
    for b in bad:
        args = dict(k=k, v=v, idx=idx)
        args.update(b)
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_gather_kv(**args)
    assert lib.calls == ["kvc_gather_kv"] * 2


def test_gather_varlen_and_hidden_checks(lib):
    total, Hkv, d, B, kk, D = 600, 2, 64, 3, 20, 256
    k = torch.empty((total, Hkv, d), dtype=bf)
    cu = torch.tensor([0, 200, 400, 600], dtype=i32)
    kvc.kvc_gather_kv_varlen(k, None, cu, torch.empty((B, Hkv, kk), dtype=i32))
    for b in (dict(idx=torch.empty((B, Hkv + 1, kk), dtype=i32)), dict(cu_seqlens=cu[:3]),
              dict(k_out=torch.empty((B, Hkv, kk, d), dtype=f32)),
              dict(idx=torch.empty((B, kk, Hkv), dtype=i32).transpose(1, 2))):
        args = dict(k=k, v=None, cu_seqlens=cu, idx=torch.empty((B, Hkv, kk), dtype=i32))
        args.update(b)
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_gather_kv_varlen(**args)
    x = torch.empty((total, D), dtype=bf)
    out = kvc.kvc_gather_hidden(x, torch.empty((1, kk), dtype=i32))
    assert tuple(out.shape) == (kk, D)
    for b in (dict(out=torch.empty((kk + 1, D), dtype=bf)), dict(idx=torch.empty(2 * kk, dtype=i32)[::2]),
              dict(x=torch.empty((total, D, 1), dtype=bf))):
        args = dict(x=x, idx=torch.empty(kk, dtype=i32))
        args.update(b)
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_gather_hidden(**args)
    assert lib.calls == ["kvc_gather_kv_varlen", "kvc_gather_hidden"]


def test_stats_checks(lib):
    rows, n = 4, 300
    S = torch.empty((rows, n), dtype=f32)
    assert tuple(kvc.kvc_layer_stats(S, 1.0).shape) == (rows, 3)
    for b in (dict(out=torch.empty((rows, 4), dtype=f32)), dict(n=n + 1),
              dict(scores=torch.empty((rows, n), dtype=torch.float64))):
        args = dict(scores=S, mass_norm=1.0)
        args.update(b)
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_layer_stats(**args)
    assert lib.calls == ["kvc_layer_stats"]


def test_pivot_update_checks(lib):
    stats = torch.empty((8, 3), dtype=f32)
    state = torch.zeros(3, dtype=torch.int64)
    kvc.kvc_pivot_update(stats, 1, 0.1, 2, 10, state)
    for b in (dict(stats=torch.empty((8, 4), dtype=f32)), dict(stats=torch.empty((3, 8), dtype=f32).t()),
              dict(state=torch.zeros(2, dtype=torch.int64)), dict(state=torch.zeros(6, dtype=torch.int32)),
              dict(stats=torch.empty((8, 3), dtype=torch.float64))):
        args = dict(stats=stats, layer=1, tau=0.1, l_min=2, l_max=10, state=state)
        args.update(b)
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_pivot_update(**args)
    assert lib.calls == ["kvc_pivot_update"]



def test_decode_checks(lib):
    H, Hkv, d, kk = 8, 2, 64, 50
    q = torch.empty((H, d), dtype=bf)
    kc, vc = torch.empty((Hkv, kk, d), dtype=bf), torch.empty((Hkv, kk, d), dtype=bf)
    ok = dict(out=torch.empty((H, d), dtype=f32), ws=_ws(), dev_err=torch.zeros(1, dtype=i32))
    out = kvc.kvc_decode_attention(q, kc, vc, **ok)
    assert out is ok["out"] and lib.calls == ["kvc_decode_attention"]
    bad_inputs = [(torch.empty((H, d + 8), dtype=bf), kc, vc),                       # head_dim differs
                  (q, kc, torch.empty((Hkv, kk + 1, d), dtype=bf)),                  # V rows differ
                  (q, torch.empty((Hkv, 2 * kk, d), dtype=bf)[:, ::2], vc),           # not contiguous
                  (q.float(), kc, vc)]                                                # not bf16
    for qq, kk_, vv in bad_inputs:
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_decode_attention(qq, kk_, vv, **ok)
    for b in (dict(out=torch.empty((H, d), dtype=torch.float64)), dict(out=torch.empty((H + 1, d), dtype=f32)),
              dict(dev_err=torch.zeros(1, dtype=torch.int64)), dict(ws=torch.empty(32, dtype=torch.uint8)[::2])):
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_decode_attention(q, kc, vc, **{**ok, **b})
    assert lib.calls == ["kvc_decode_attention"]


def test_prefill_checks(lib):
    n, H, Hkv, d = 20, 8, 2, 64
    q = torch.empty((n, H, d), dtype=bf)
    k, v = torch.empty((n, Hkv, d), dtype=bf), torch.empty((n, Hkv, d), dtype=bf)
    out, lse = kvc.kvc_prefill_attention(q, k, v, dev_err=torch.zeros(1, dtype=i32))
    assert tuple(out.shape) == (n, H, d) and out.dtype == bf
    assert tuple(lse.shape) == (n, H) and lse.dtype == f32
    out2, _ = kvc.kvc_prefill_attention(q, k, v, want_out=False)
    assert out2 is None and lib.calls == ["kvc_prefill_attention"] * 2
    bad_inputs = [(q, torch.empty((n + 1, Hkv, d), dtype=bf), v),                   # rows differ
                  (q, k, torch.empty((n, Hkv + 1, d), dtype=bf)),                    # V heads differ
                  (q, torch.empty((n, Hkv, d + 8), dtype=bf), v),                    # head_dim differs
                  (torch.empty((n, 2 * H, d), dtype=bf)[:, ::2], k, v)]              # not contiguous
    for qq, kk_, vv in bad_inputs:
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_prefill_attention(qq, kk_, vv)
    for b in (dict(out=torch.empty((n, H, d + 1), dtype=bf)), dict(out=torch.empty((n, H, d), dtype=f32)),
              dict(lse=torch.empty((n, H), dtype=torch.float64)), dict(lse=torch.empty((H, n), dtype=f32)),
              dict(dev_err=torch.zeros(1, dtype=torch.int64))):
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_prefill_attention(q, k, v, **b)
    assert lib.calls == ["kvc_prefill_attention"] * 2


def test_rvq_checks(lib):
    n, d, S, M = 30, 64, 3, 16
    x, cb = torch.empty((n, d), dtype=bf), torch.empty((S, M, d), dtype=f32)
    codes, res = kvc.kvc_rvq_encode(x, cb, residual=torch.empty((n, d), dtype=f32))
    assert tuple(codes.shape) == (n, S) and codes.dtype == i32 and tuple(res.shape) == (n, d)
    codes, res = kvc.kvc_rvq_encode(x, cb)
    assert res is None and lib.calls == ["kvc_rvq_encode"] * 2
    for bad_cb in (torch.empty((S, M, d), dtype=torch.float64), torch.empty((S, M, d + 1), dtype=f32),
                   torch.empty((S, d, M), dtype=f32).transpose(1, 2), torch.empty((M, d), dtype=f32)):
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_rvq_encode(x, bad_cb)
    for b in (dict(codes=torch.empty((n, S + 1), dtype=i32)), dict(codes=torch.empty((n, S), dtype=torch.int64)),
              dict(residual=torch.empty((n, d + 1), dtype=f32)), dict(dev_err=torch.zeros(1, dtype=torch.int64))):
        with pytest.raises((ValueError, TypeError)):
            kvc.kvc_rvq_encode(x, cb, **b)
    with pytest.raises((ValueError, TypeError)):
        kvc.kvc_rvq_encode(x.float(), cb)
    assert lib.calls == ["kvc_rvq_encode"] * 2
