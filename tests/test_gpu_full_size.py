"""Parity at the full sizes of the benchmark configurations, in the launch
configuration the benchmark times: the 128K layer with TSP and hidden-state
gather, the ragged batch of eight sequences, and the sixteen-layer
accumulation.  Whole score rows and whole index sets are compared with the
float64 oracle (scores within the relative tolerance, index sets under the
near-tie band rule); gathers are bit-exact against plain indexing."""
import numpy as np
import pytest
import torch

import long_context_kv_window_b200 as kvc
import oracle
import workloads
from tests import parity
from tests.gpu_helpers import dev_bf16, host_bits

pytestmark = pytest.mark.gpu


def test_c3_full_layer_through_layer_plan():
    """N = 131072, 32 query / 8 KV heads, window 32, pool 7, K/V budget
    13107 per head, TSP budget 26214, hidden 4096: every output."""
    cfg = workloads.C3
    lay = workloads.make_layer(cfg)
    q, k, v, x = (dev_bf16(a) for a in (lay.q, lay.k, lay.v, lay.x))
    plan = kvc.LayerPlan(cfg.N, cfg.H, cfg.Hkv, cfg.d, cfg.w, cfg.k_kv, cfg.k_tsp, cfg.hidden, True, "cuda",
                         pool_kernel=cfg.pool)
    out = plan.run(q, k, v, x)
    # the same layer with the scoring call writing the head-sum row, which the TSP selection then ranks
    plan_row = kvc.LayerPlan(cfg.N, cfg.H, cfg.Hkv, cfg.d, cfg.w, cfg.k_kv, cfg.k_tsp, cfg.hidden, True, "cuda",
                             pool_kernel=cfg.pool, tsp_row=True)
    out_row = plan_row.run(q, k, v, x)
    torch.cuda.synchronize()
    assert plan.dev_err.item() == 0
    res = oracle.layer(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale, cfg.pool, cfg.k_kv, cfg.k_tsp)

    err = parity.assert_scores_close(out.scores.cpu().numpy(), res.A, what="c3 scores")
    idx = out.idx_kv.cpu().numpy()
    for g in range(cfg.Hkv):
        parity.assert_selection_matches(idx[g], res.idx_kv[g], res.pooled[g], cfg.N, cfg.w, cfg.k_kv,
                                        what=f"c3 head {g}")
    parity.assert_scores_close(out_row.tsp[0].cpu().numpy(), res.T, what="c3 head-sum row")
    it = out.idx_tsp[0].cpu().numpy()
    assert np.array_equal(it, out_row.idx_tsp[0].cpu().numpy()), "TSP set: summed on the fly vs the head-sum row"
    parity.assert_selection_matches(it, res.idx_tsp, res.pooled_tsp, cfg.N, cfg.w, cfg.k_tsp, what="c3 TSP set")

    kc, vc = host_bits(out.k_c), host_bits(out.v_c)
    for g in range(cfg.Hkv):
        assert np.array_equal(kc[g], lay.k[idx[g], g, :]), f"K gather head {g}"
        assert np.array_equal(vc[g], lay.v[idx[g], g, :]), f"V gather head {g}"
    assert np.array_equal(host_bits(out.x_c), lay.x[it]), "hidden gather"
    print(f"c3: max score rel err {err:.2e}")


def test_c4_full_ragged_batch():
    """Eight sequences of U[4096, 65536] tokens packed (about 3e5), budget
    1024 per head and sequence: every sequence against its own oracle run."""
    cfg = workloads.C4
    lay = workloads.make_layer(cfg)
    B, w = lay.batch, cfg.w
    q = dev_bf16(lay.q).view(B, w, cfg.H, cfg.d)
    k, v = dev_bf16(lay.k), dev_bf16(lay.v)
    cu = torch.from_numpy(lay.cu_seqlens.astype(np.int32)).cuda()
    max_len = int(lay.lengths().max())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    scores = kvc.kvc_score_varlen(q, k, cu, max_len, dev_err=err)
    idx, counts = kvc.kvc_select_topk_varlen(scores, cu, max_len, w, cfg.pool, cfg.k_kv, dev_err=err)
    kc, vc = kvc.kvc_gather_kv_varlen(k, v, cu, idx, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    S, I = scores.cpu().numpy(), idx.cpu().numpy()
    KC, VC = host_bits(kc), host_bits(vc)
    cuh = lay.cu_seqlens
    assert np.array_equal(counts.cpu().numpy(), np.minimum(cfg.k_kv, np.diff(cuh)))
    for b in range(B):
        s0, s1 = int(cuh[b]), int(cuh[b + 1])
        n = s1 - s0
        res = oracle.layer(lay.q[b * w:(b + 1) * w], lay.k[s0:s1], cfg.H, cfg.Hkv, w, cfg.scale, cfg.pool,
                           cfg.k_kv)
        parity.assert_scores_close(S[:, s0:s1], res.A, what=f"c4 sequence {b} scores")
        m = min(cfg.k_kv, n)
        for g in range(cfg.Hkv):
            parity.assert_selection_matches(I[b, g, :m], res.idx_kv[g], res.pooled[g], n, w, cfg.k_kv,
                                            what=f"c4 sequence {b} head {g}")
            rows = s0 + I[b, g, :m]
            assert np.array_equal(KC[b, g, :m], lay.k[rows, g, :])
            assert np.array_equal(VC[b, g, :m], lay.v[rows, g, :])


def test_c5_full_sixteen_layers():
    """Sixteen layers of N = 65536 with 40 query / 8 KV heads (160 window rows
    per KV head), no pooling, all eight KV heads.  C_global (the sum of the
    per-layer scores, accumulated by the scoring call) is compared after the
    last layer, and both of that layer's selections rank C_global: the
    propagation set of 15 % of the tokens over the sum of the eight rows
    (9830 kept) and the 4096-per-KV-head K set.  The last layer's own scores
    and statistics are compared too."""
    cfg = workloads.C5
    N, G, w, Hkv = cfg.N, cfg.G, cfg.w, cfg.Hkv
    orc = oracle.get()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    accum = torch.zeros((Hkv, N), dtype=torch.float32, device="cuda")
    ref_c = np.zeros((Hkv, N))
    A = None
    for layer in range(1, cfg.layers + 1):
        lay = workloads.make_layer(cfg, layer=layer)
        scores = kvc.kvc_score(dev_bf16(lay.q), dev_bf16(lay.k), accum=accum, dev_err=err)
        A = orc.window_scores(lay.q, lay.k, cfg.H, Hkv, w, cfg.scale)
        ref_c += A
    idx_prop = kvc.kvc_select_topk(accum, w, cfg.pool, cfg.k_tsp, row_group=Hkv)
    idx_kv = kvc.kvc_select_topk(accum, w, cfg.pool, cfg.k_kv)
    stats = kvc.kvc_layer_stats(scores, float(w * G))
    torch.cuda.synchronize()
    assert err.item() == 0
    parity.assert_scores_close(accum.cpu().numpy(), ref_c, what="c5 C_global")
    parity.assert_scores_close(scores.cpu().numpy(), A, what="c5 last-layer scores")
    T = orc.sum_rows(ref_c)
    S_prop = orc.rank_scores(T, N, w, cfg.pool)
    parity.assert_selection_matches(idx_prop[0].cpu().numpy(), orc.select_topk(S_prop, N, w, cfg.k_tsp), S_prop,
                                    N, w, cfg.k_tsp, what="c5 propagation set (C_global, all heads)")
    ik = idx_kv.cpu().numpy()
    st = stats.cpu().numpy()
    for g in range(Hkv):
        S = orc.rank_scores(ref_c[g], N, w, cfg.pool)
        parity.assert_selection_matches(ik[g], orc.select_topk(S, N, w, cfg.k_kv), S, N, w, cfg.k_kv,
                                        what=f"c5 K set of head {g} (C_global)")
        parity.assert_scores_close(st[g], orc.layer_stats(A[g], w * G), what=f"c5 last-layer stats head {g}")
