"""CPU tests of the C-ABI boundary: the library loads, exports every entry
point that include/kvc.h declares, and rejects bad arguments on the host
before touching the GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

import long_context_kv_window_b200 as kvc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvc.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(kvc_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from long_context_kv_window_b200 import build
    build.build()
    return kvc.lib()


def test_header_declares_the_documented_calls():
    names = declared_functions()
    for must in ("kvc_score", "kvc_select_topk", "kvc_gather_kv", "kvc_gather_hidden", "kvc_score_varlen",
                 "kvc_select_topk_varlen", "kvc_gather_kv_varlen", "kvc_layer_stats"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"
    for n in names:
        assert n in kvc._SIGS, f"no binding signature for {n}"


def test_version_and_status_strings(lib):
    assert kvc.abi_version() == 1
    assert kvc.status_string(0) == "KVC_OK"
    assert kvc.status_string(1) == "KVC_ERR_INVALID_ARG"
    assert kvc.status_string(99) == "KVC_ERR_UNKNOWN"


def _p(H=8, Hkv=2, d=64, w=8, scale=0.125):
    return kvc.ScoreParams(H, Hkv, d, w, scale)


def test_workspace_sizes_are_host_only(lib):
    n = ctypes.c_size_t()
    assert lib.kvc_score_workspace_size(ctypes.byref(_p()), 1, 512, ctypes.byref(n)) == 0
    assert n.value > 0
    big = ctypes.c_size_t()
    assert lib.kvc_score_workspace_size(ctypes.byref(_p(32, 8, 128, 32)), 8, 300000, ctypes.byref(big)) == 0
    assert big.value > n.value
    assert lib.kvc_select_workspace_size(8, 1, 131072, ctypes.byref(n)) == 0
    assert n.value >= 8 * 131072 * 4


@pytest.mark.parametrize("params,status", [
    (dict(d=96), 2),              # unsupported head dim
    (dict(H=6, Hkv=4), 1),        # H % Hkv != 0
    (dict(w=0), 1),               # empty window
    (dict(H=16, Hkv=1, w=32), 2),  # G * w > 256
    (dict(scale=0.0), 1),
])
def test_score_rejects_bad_params_before_launch(lib, params, status):
    ws = ctypes.c_size_t()
    before = kvc.launch_count()
    rc = lib.kvc_score_workspace_size(ctypes.byref(_p(**params)), 1, 512, ctypes.byref(ws))
    assert rc == status
    assert kvc.last_error() != ""
    assert kvc.launch_count() == before


def test_null_pointers_and_bad_sizes_are_rejected(lib):
    dummy = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    p = _p()
    assert lib.kvc_score(None, 512, 64, dummy, 128, 64, 512, ctypes.byref(p), dummy, None, None, dummy,
                         1 << 20, None, None) == 1
    # n < window
    assert lib.kvc_score(dummy, 512, 64, dummy, 128, 64, 4, ctypes.byref(p), dummy, None, None, dummy,
                         1 << 20, None, None) == 1
    # misaligned stride (not a multiple of 8 elements)
    assert lib.kvc_score(dummy, 512, 64, dummy, 130, 64, 512, ctypes.byref(p), dummy, None, None, dummy,
                         1 << 20, None, None) == 1
    # workspace too small
    assert lib.kvc_score(dummy, 512, 64, dummy, 128, 64, 512, ctypes.byref(p), dummy, None, None, dummy,
                         16, None, None) == 4
    # select: k < window, even pool kernel, rows not a multiple of row_group
    assert lib.kvc_select_topk(dummy, 2, 512, 1, 512, 8, 1, 4, dummy, 64, None, dummy, 1 << 20, None) == 1
    assert lib.kvc_select_topk(dummy, 2, 512, 1, 512, 8, 4, 64, dummy, 64, None, dummy, 1 << 20, None) == 1
    assert lib.kvc_select_topk(dummy, 3, 512, 2, 512, 8, 1, 64, dummy, 64, None, dummy, 1 << 20, None) == 1
    # gathers: head_dim 80 unsupported, hidden not a multiple of 8, misaligned pointer
    assert lib.kvc_gather_kv(dummy, None, 160, 80, 512, 2, 80, dummy, 64, 64, dummy, None, None, None) == 2
    assert lib.kvc_gather_hidden(dummy, 4100, 512, 4100, dummy, 10, dummy, None, None) == 1
    odd = ctypes.c_void_p(258)
    assert lib.kvc_gather_hidden(odd, 4096, 512, 4096, dummy, 10, dummy, None, None) == 1
    # varlen: batch out of range
    assert lib.kvc_score_varlen(dummy, 4096, 512, 64, dummy, 128, 64, dummy, 0, 512, 512, ctypes.byref(p),
                                dummy, None, None, dummy, 1 << 20, None, None) == 1
    assert lib.kvc_layer_stats(dummy, 2, 512, 512, 0.0, dummy, None, 0, None) == 1


def test_given_normaliser_and_pivot_calls_reject_bad_arguments(lib):
    dummy = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    p = _p()
    before = kvc.launch_count()
    # kvc_score_lse: NULL lse, negative lse stride, n < window, workspace too small
    assert lib.kvc_score_lse(dummy, 512, 64, dummy, 128, 64, 512, ctypes.byref(p), None, 1, 512, dummy, None, None,
                             dummy, 1 << 20, None, None) == 1
    assert lib.kvc_score_lse(dummy, 512, 64, dummy, 128, 64, 512, ctypes.byref(p), dummy, -1, 512, dummy, None,
                             None, dummy, 1 << 20, None, None) == 1
    assert lib.kvc_score_lse(dummy, 512, 64, dummy, 128, 64, 4, ctypes.byref(p), dummy, 1, 512, dummy, None, None,
                             dummy, 1 << 20, None, None) == 1
    assert lib.kvc_score_lse(dummy, 512, 64, dummy, 128, 64, 512, ctypes.byref(p), dummy, 1, 512, dummy, None, None,
                             dummy, 16, None, None) == 4
    # kvc_pivot_update: NULL stats, rows 0, layer 0, tau < 0, l_max < l_min, misaligned state
    state = ctypes.c_void_p(512)
    assert lib.kvc_pivot_update(None, 8, 1, 0.1, 1, 4, state, None, None) == 1
    assert lib.kvc_pivot_update(dummy, 0, 1, 0.1, 1, 4, state, None, None) == 1
    assert lib.kvc_pivot_update(dummy, 8, 0, 0.1, 1, 4, state, None, None) == 1
    assert lib.kvc_pivot_update(dummy, 8, 1, -0.1, 1, 4, state, None, None) == 1
    assert lib.kvc_pivot_update(dummy, 8, 1, 0.1, 5, 4, state, None, None) == 1
    assert lib.kvc_pivot_update(dummy, 8, 1, 0.1, 1, 4, ctypes.c_void_p(516), None, None) == 1
    assert kvc.last_error() != ""
    assert kvc.launch_count() == before


def test_decode_attention_rejects_bad_arguments(lib):
    dummy = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    before = kvc.launch_count()
    n = ctypes.c_size_t()
    assert lib.kvc_decode_workspace_size(32, 8, 128, 13107, ctypes.byref(n)) == 0 and n.value > 0
    assert lib.kvc_decode_workspace_size(32, 8, 96, 13107, ctypes.byref(n)) == 2      # head_dim 96
    assert lib.kvc_decode_workspace_size(32, 8, 128, 0, ctypes.byref(n)) == 1         # no entries
    assert lib.kvc_decode_workspace_size(34, 2, 128, 100, ctypes.byref(n)) == 2       # 17 heads per KV head
    assert lib.kvc_decode_workspace_size(30, 8, 128, 100, ctypes.byref(n)) == 1       # H not a multiple of Hkv
    ws = 1 << 20
    # NULL out, misaligned k_c, q stride below head_dim, zero scale, workspace too small
    assert lib.kvc_decode_attention(dummy, 128, dummy, dummy, 100, 32, 8, 128, 0.1, None, dummy, ws, None, None) == 1
    assert lib.kvc_decode_attention(dummy, 128, ctypes.c_void_p(264), dummy, 100, 32, 8, 128, 0.1, dummy, dummy, ws,
                                    None, None) == 1
    assert lib.kvc_decode_attention(dummy, 64, dummy, dummy, 100, 32, 8, 128, 0.1, dummy, dummy, ws, None, None) == 1
    assert lib.kvc_decode_attention(dummy, 128, dummy, dummy, 100, 32, 8, 128, 0.0, dummy, dummy, ws, None, None) == 1
    assert lib.kvc_decode_attention(dummy, 128, dummy, dummy, 100, 32, 8, 128, 0.1, dummy, dummy, 16, None, None) == 4
    assert kvc.launch_count() == before


def test_prefill_attention_rejects_bad_arguments(lib):
    dummy = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    before = kvc.launch_count()
    assert lib.kvc_prefill_attention(None, dummy, dummy, 100, 32, 8, 128, 0.1, dummy, dummy, None, None) == 1
    assert lib.kvc_prefill_attention(dummy, dummy, dummy, 100, 32, 8, 64, 0.1, dummy, dummy, None, None) == 2  # d 64
    assert lib.kvc_prefill_attention(dummy, dummy, dummy, 100, 30, 8, 128, 0.1, dummy, dummy, None, None) == 1
    assert lib.kvc_prefill_attention(dummy, dummy, dummy, 0, 32, 8, 128, 0.1, dummy, dummy, None, None) == 1
    assert lib.kvc_prefill_attention(dummy, dummy, dummy, 100, 32, 8, 128, 0.0, dummy, dummy, None, None) == 1
    assert lib.kvc_prefill_attention(dummy, ctypes.c_void_p(264), dummy, 100, 32, 8, 128, 0.1, dummy, dummy,
                                     None, None) == 1  # misaligned k
    assert kvc.last_error() != ""
    assert kvc.launch_count() == before


def test_rvq_encode_rejects_bad_arguments(lib):
    dummy = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    before = kvc.launch_count()
    assert lib.kvc_rvq_encode(dummy, 128, 10, 96, dummy, 4, 256, dummy, None, None, None) == 2   # head_dim 96
    assert lib.kvc_rvq_encode(dummy, 128, 10, 128, dummy, 4, 300, dummy, None, None, None) == 2  # M > 256
    assert lib.kvc_rvq_encode(dummy, 128, 10, 128, dummy, 4, 40, dummy, None, None, None) == 2   # M % 16
    assert lib.kvc_rvq_encode(dummy, 128, 10, 128, dummy, 0, 256, dummy, None, None, None) == 1  # no stage
    assert lib.kvc_rvq_encode(dummy, 64, 10, 128, dummy, 4, 256, dummy, None, None, None) == 1   # stride < d
    assert lib.kvc_rvq_encode(dummy, 128, 10, 128, ctypes.c_void_p(260), 4, 256, dummy, None, None, None) == 1
    assert lib.kvc_rvq_encode(dummy, 128, 10, 128, dummy, 4, 256, None, None, None, None) == 1   # NULL codes
    assert lib.kvc_rvq_encode(dummy, 128, 0, 128, dummy, 4, 256, dummy, None, None, None) == 0   # nothing to do
    assert kvc.launch_count() == before
