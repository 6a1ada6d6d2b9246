"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs.  Scores within relative 1e-3, index sets identical
up to the near-tie band, gathers bit-exact (see tests/parity.py)."""
import math

import numpy as np
import pytest
import torch

import long_context_kv_window_b200 as kvc
import oracle
import workloads
from tests import oracle_pins, parity
from tests.gpu_helpers import check_layer, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvc.lib()  # fail loudly if the library is missing
    torch.cuda.set_device(0)


def _err_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# --------------------------------------------------------------------------- #
# gathers
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("d", [64, 128])
def test_gather_kv_bit_exact(d):
    rng = np.random.default_rng(5)
    N, Hkv, kk = 777, 3, 100
    k = rng.integers(0, 1 << 16, size=(N, Hkv, d), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(N, Hkv, d), dtype=np.uint16)
    idx = np.sort(rng.choice(N, size=(Hkv, kk), replace=True), axis=1).astype(np.int32)
    idx[1, 5] = -1
    err = _err_word()
    ko, vo = kvc.kvc_gather_kv(dev_bf16(k), dev_bf16(v), torch.from_numpy(idx).cuda(), dev_err=err)
    orc = oracle.get()
    ref_k, bad_k = orc.gather_kv(k, idx)
    ref_v, _ = orc.gather_kv(v, idx)
    assert bad_k == 0 and err.item() == 0
    assert np.array_equal(host_bits(ko), ref_k) and np.array_equal(host_bits(vo), ref_v)
    # out-of-range indices: zero rows and the device error bit
    idx[0, 0] = N
    idx[2, 3] = -5
    ko, vo = kvc.kvc_gather_kv(dev_bf16(k), dev_bf16(v), torch.from_numpy(idx).cuda(), dev_err=err)
    ref_k, bad = orc.gather_kv(k, idx)
    assert bad == 2 and err.item() == kvc.KVC_DEV_ERR_INDEX
    assert np.array_equal(host_bits(ko), ref_k)


def test_gather_kv_broadcast_index_row():
    rng = np.random.default_rng(6)
    N, Hkv, d, kk = 300, 4, 128, 37
    k = rng.integers(0, 1 << 16, size=(N, Hkv, d), dtype=np.uint16)
    idx = np.sort(rng.choice(N, size=kk, replace=False)).astype(np.int32)
    ko, vo = kvc.kvc_gather_kv(dev_bf16(k), None, torch.from_numpy(idx[None]).cuda())
    assert vo is None
    ref, _ = oracle.get().gather_kv(k, np.tile(idx, (Hkv, 1)))
    assert np.array_equal(host_bits(ko), ref)


@pytest.mark.parametrize("D", [4096, 1000, 8])
def test_gather_hidden_bit_exact(D):
    rng = np.random.default_rng(7)
    N, kk = 513, 200
    x = rng.integers(0, 1 << 16, size=(N, D), dtype=np.uint16)
    idx = rng.integers(-1, N, size=kk).astype(np.int32)
    err = _err_word()
    out = kvc.kvc_gather_hidden(dev_bf16(x), torch.from_numpy(idx).cuda(), dev_err=err)
    ref, bad = oracle.get().gather_rows(x, idx)
    assert bad == 0 and err.item() == 0
    assert np.array_equal(host_bits(out), ref)


# --------------------------------------------------------------------------- #
# selection on given scores
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("n,w,k,levels", [(50, 5, 12, 50), (1000, 8, 64, 50), (4097, 32, 1000, 50),
                                          (20000, 32, 2048, 50), (300, 10, 10, 50), (300, 10, 300, 50),
                                          (300, 10, 1000, 50), (131072, 32, 13107, 50),
                                          (131072, 32, 13107, 3), (131072, 32, 70000, 1)])
def test_select_exact_on_given_scores_no_pool(n, w, k, levels):
    """Without pooling the GPU ranks exactly the values the oracle ranks: the
    sets must be identical (ties included: many repeated values).  With 3 or 1
    distinct values the threshold bin of the first radix digit holds tens of
    thousands of keys, more than the candidate list takes, so the remaining
    digits run cluster-wide."""
    rng = np.random.default_rng(n + k)
    S = rng.integers(0, levels, size=(3, n)).astype(np.float32) * 0.25
    idx = kvc.kvc_select_topk(torch.from_numpy(S).cuda(), w, 1, k).cpu().numpy()
    orc = oracle.get()
    for r in range(3):
        ref = orc.select_topk(S[r, : n - w].astype(np.float64), n, w, k)
        assert np.array_equal(idx[r], ref), f"row {r}"


def test_select_window_miss_falls_back_to_plain_radix():
    """The selection brackets the k-th largest key with a window taken from
    a sample of each CTA's keys (evenly spaced positions).  Here exactly the
    sampled positions hold large values and everything else small ones, so the
    window lands far above the true threshold; the result must still be exact
    (the kernel then ranks with a plain radix select)."""
    n, w, k, rows = 200000, 32, 20000, 4
    L = n - w
    cs = 8
    seg = ((L + cs - 1) // cs + 3) & ~3
    rng = np.random.default_rng(11)
    S = rng.random((rows, n)).astype(np.float32)
    for c in range(cs):
        s0 = min(c * seg, L)
        nseg = min(seg, L - s0)
        nsc = min(256 // cs, nseg)
        pos = s0 + ((2 * np.arange(nsc) + 1) * nseg) // (2 * nsc)
        S[:, pos] = 100.0 + rng.random((rows, nsc)).astype(np.float32)
    idx = kvc.kvc_select_topk(torch.from_numpy(S).cuda(), w, 1, k).cpu().numpy()
    orc = oracle.get()
    for r in range(rows):
        ref = orc.select_topk(S[r, :L].astype(np.float64), n, w, k)
        assert np.array_equal(idx[r], ref), f"row {r}"


@pytest.mark.parametrize("case", ["levels50", "levels3", "levels1", "lognormal_pool7", "window_miss",
                                  "uniform_pool7_n65536"])
def test_select_single_long_row_wide_cluster(case):
    """A lone ranking row of 32K positions or more (the all-head TSP row) is
    spread over a 16-CTA cluster where the device can place one.  It must
    rank like the oracle and exactly like the 8-CTA launch of the same row
    (two identical rows in one call take the 8-CTA path)."""
    rng = np.random.default_rng(abs(hash(case)) % 2**32)
    n, w, k, pool = 131072, 32, 26214, 1
    if case.startswith("levels"):
        S = rng.integers(0, int(case[6:]), size=n).astype(np.float32) * 0.25
    elif case == "lognormal_pool7":
        S, pool = np.exp(3.0 * rng.standard_normal(n)).astype(np.float32), 7
    elif case == "window_miss":
        # the evenly spaced positions each CTA samples hold large values
        L, cs = n - w, 16
        seg = ((L + cs - 1) // cs + 3) & ~3
        S = rng.random(n).astype(np.float32)
        for c in range(cs):
            s0 = min(c * seg, L)
            nseg = min(seg, L - s0)
            nsc = min(128 // cs, nseg)
            S[s0 + ((2 * np.arange(nsc) + 1) * nseg) // (2 * nsc)] = 100.0 + rng.random(nsc).astype(np.float32)
    else:
        n, k, pool = 65536, 9830, 7
        S = rng.random(n).astype(np.float32)
    one = torch.from_numpy(S).view(1, n).cuda()
    idx1 = kvc.kvc_select_topk(one, w, pool, k).cpu().numpy()[0]
    idx8 = kvc.kvc_select_topk(one.expand(2, n).contiguous(), w, pool, k).cpu().numpy()
    assert np.array_equal(idx1, idx8[0]) and np.array_equal(idx1, idx8[1]), "16-CTA and 8-CTA launches differ"
    orc = oracle.get()
    Sp = orc.rank_scores(S.astype(np.float64), n, w, pool)
    ref = orc.select_topk(Sp, n, w, k)
    if pool == 1:
        assert np.array_equal(idx1, ref)
    else:
        parity.assert_selection_matches(idx1, ref, Sp, n, w, k)


@pytest.mark.parametrize("n,pool", [(420000, 7), (420000, 1)])
def test_select_long_row_global_memory_mode(n, pool):
    """Rows too long for the per-CTA shared-memory segments: pooled values
    live in global memory during ranking and are averages on return."""
    rng = np.random.default_rng(n + pool)
    w, k = 32, 4200
    S = (rng.random((2, n)) ** 4).astype(np.float32)
    pooled = torch.empty((2, n - w), dtype=torch.float32, device="cuda")
    idx = kvc.kvc_select_topk(torch.from_numpy(S).cuda(), w, pool, k, pooled=pooled).cpu().numpy()
    idx_ws = kvc.kvc_select_topk(torch.from_numpy(S).cuda(), w, pool, k).cpu().numpy()
    assert np.array_equal(idx, idx_ws)
    orc = oracle.get()
    for r in range(2):
        Sp = orc.rank_scores(S[r].astype(np.float64), n, w, pool)
        parity.assert_scores_close(pooled[r].cpu().numpy(), Sp, rtol=1e-6, what="pooled")
        parity.assert_selection_matches(idx[r], orc.select_topk(Sp, n, w, k), Sp, n, w, k)


@pytest.mark.parametrize("pool", [1, 3, 7, 9, 11, 65])
def test_select_pooled_and_grouped(pool):
    rng = np.random.default_rng(pool)
    n, w, k, rows, grp = 9000, 16, 700, 8, 4
    S = (rng.random((rows, n)) ** 4).astype(np.float32)
    pooled = torch.empty((rows // grp, n - w), dtype=torch.float32, device="cuda")
    idx = kvc.kvc_select_topk(torch.from_numpy(S).cuda(), w, pool, k, row_group=grp, pooled=pooled)
    idx = idx.cpu().numpy()
    orc = oracle.get()
    for o in range(rows // grp):
        T = orc.sum_rows(S[o * grp:(o + 1) * grp].astype(np.float64))
        Sp = orc.rank_scores(T, n, w, pool)
        ref = orc.select_topk(Sp, n, w, k)
        parity.assert_scores_close(pooled[o].cpu().numpy(), Sp, rtol=1e-6, what="pooled")
        parity.assert_selection_matches(idx[o], ref, Sp, n, w, k)


@pytest.mark.parametrize("grp", [2, 3, 5, 7, 8, 16])
def test_select_row_groups_of_every_size(grp):
    """Row-group sums formed while staging, for group sizes that take each
    load-batching shape of the staging (8, 4 or 2 rows per batch of loads,
    with a partial last batch for 3, 5 and 7 rows): two output rows, each
    the pooled sum of its group, against the oracle's sums."""
    rng = np.random.default_rng(100 + grp)
    n, w, k, pool = 5000, 16, 400, 7
    rows = 2 * grp
    S = (rng.random((rows, n)) ** 4).astype(np.float32)
    pooled = torch.empty((2, n - w), dtype=torch.float32, device="cuda")
    idx = kvc.kvc_select_topk(torch.from_numpy(S).cuda(), w, pool, k, row_group=grp, pooled=pooled).cpu().numpy()
    orc = oracle.get()
    for o in range(2):
        T = orc.sum_rows(S[o * grp:(o + 1) * grp].astype(np.float64))
        Sp = orc.rank_scores(T, n, w, pool)
        parity.assert_scores_close(pooled[o].cpu().numpy(), Sp, rtol=1e-6, what=f"pooled, groups of {grp}")
        parity.assert_selection_matches(idx[o], orc.select_topk(Sp, n, w, k), Sp, n, w, k)


# --------------------------------------------------------------------------- #
# scoring + selection + gathers on the configurations
# --------------------------------------------------------------------------- #
def _run_layer(lay, cfg, k_kv=None, k_tsp=None):
    q = dev_bf16(lay.q)
    kd = dev_bf16(lay.k)
    vd = dev_bf16(lay.v) if lay.v is not None else None
    N = lay.k.shape[0]
    err = _err_word()
    tsp = torch.empty(N, dtype=torch.float32, device="cuda") if k_tsp else None
    scores = kvc.kvc_score(q, kd, tsp=tsp, dev_err=err)
    idx = kvc.kvc_select_topk(scores, cfg.w, cfg.pool, k_kv or cfg.k_kv)
    ko, vo = kvc.kvc_gather_kv(kd, vd, idx, dev_err=err)
    out = dict(scores=scores.cpu().numpy(), idx=idx.cpu().numpy(), k_c=host_bits(ko),
               v_c=host_bits(vo) if vo is not None else None, err=err.item())
    if k_tsp:
        it = kvc.kvc_select_topk(scores, cfg.w, cfg.pool, k_tsp, row_group=cfg.Hkv)
        out["tsp"] = tsp.cpu().numpy()
        out["idx_tsp"] = it.cpu().numpy()[0]
    return out


def test_tiny_config_end_to_end():
    cfg = workloads.C1
    lay = workloads.make_layer(cfg)
    g = _run_layer(lay, cfg)
    assert g["err"] == 0
    res, err, kinds = check_layer(lay, cfg, g["scores"], g["idx"], what="tiny")
    assert err < 1e-4, err
    ref_k, _ = oracle.get().gather_kv(lay.k, g["idx"])
    ref_v, _ = oracle.get().gather_kv(lay.v, g["idx"])
    assert np.array_equal(g["k_c"], ref_k) and np.array_equal(g["v_c"], ref_v)
    for gg in range(cfg.Hkv):
        assert np.all(np.isin(lay.hitters[0], g["idx"][gg]))
    assert np.allclose(g["scores"].sum(axis=1), cfg.rows, rtol=1e-5)


@pytest.mark.parametrize("N", [8, 9, 100, 127, 128, 129, 1000, 4097])
def test_tiny_heads_edge_lengths(N):
    """Tile edges, ragged tails and the window covering (almost) everything."""
    cfg = workloads.shrink(workloads.C1, N=N, n_hitters=min(4, max(0, N - 8 - 1)), k_kv=min(64, N), seed=1000 + N)
    lay = workloads.make_layer(cfg)
    g = _run_layer(lay, cfg)
    check_layer(lay, cfg, g["scores"], g["idx"], what=f"N={N}")


@pytest.mark.parametrize("N,H,Hkv,w,pool,k", [(129, 32, 8, 32, 7, 64), (300, 32, 8, 32, 7, 100),
                                                (2000, 40, 8, 32, 1, 500), (3000, 16, 2, 8, 5, 333),
                                                (5000, 8, 8, 16, 7, 999)])
def test_d128_shapes(N, H, Hkv, w, pool, k):
    cfg = workloads.shrink(workloads.C2, N=N, H=H, Hkv=Hkv, w=w, pool=pool, k_kv=k,
                           n_sinks=min(4, N - w), n_hitters=min(8, N - w - 4), seed=2000 + N)
    lay = workloads.make_layer(cfg)
    g = _run_layer(lay, cfg)
    check_layer(lay, cfg, g["scores"], g["idx"], what=f"H={H} Hkv={Hkv} N={N}")


@pytest.mark.parametrize("base,N,H,Hkv,w,pool,k", [
    ("C2", 3000, 68, 4, 8, 7, 500),   # R = 136: pass 2 three 160-column buffers, 144-row MMA (16-column tail)
    ("C2", 2500, 48, 8, 32, 3, 400),  # R = 192: two 192-column buffers in pass 2, two 256 in pass 1
    ("C2", 2000, 64, 8, 32, 1, 300),  # R = 256: the widest accumulator, 512 TMEM columns in both passes
    ("C2", 1500, 10, 2, 8, 5, 200),   # R = 40: four 64-column buffers, 48-row MMA
    ("C1", 2000, 34, 2, 8, 7, 300),   # d = 64, R = 136
])
def test_wide_window_rows(base, N, H, Hkv, w, pool, k):
    """Window row counts past one 128-row block and ragged MMA widths: the
    accumulator widths that leave room for fewer TMEM buffers (one epilogue
    group per buffer) and the 16-column tail of the column walk."""
    cfg = workloads.shrink(getattr(workloads, base), N=N, H=H, Hkv=Hkv, w=w, pool=pool, k_kv=k,
                           n_sinks=4, n_hitters=8, seed=5000 + H)
    lay = workloads.make_layer(cfg)
    g = _run_layer(lay, cfg)
    assert g["err"] == 0
    check_layer(lay, cfg, g["scores"], g["idx"], what=f"{base} H={H} Hkv={Hkv} w={w}")


def test_llama_32k_full_size():
    cfg = workloads.C2
    lay = workloads.make_layer(cfg)
    g = _run_layer(lay, cfg)
    assert g["err"] == 0
    res, err, kinds = check_layer(lay, cfg, g["scores"], g["idx"], what="32K")
    print(f"32K: max score rel err {err:.2e}, selection kinds {kinds}")
    for gg in range(cfg.Hkv):
        assert np.all(np.isin(lay.sinks[0], g["idx"][gg]))
        assert np.all(np.isin(lay.hitters[0], g["idx"][gg]))
    ref_k, _ = oracle.get().gather_kv(lay.k, g["idx"])
    assert np.array_equal(g["k_c"], ref_k)


def test_tsp_aggregate_and_selection():
    cfg = workloads.shrink(workloads.C3, N=20000, k_kv=2000, k_tsp=4000, hidden=None, n_hitters=32, seed=3001)
    lay = workloads.make_layer(cfg, with_x=False)
    g = _run_layer(lay, cfg, k_tsp=cfg.k_tsp)
    res = oracle.layer(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale, cfg.pool, cfg.k_kv, k_tsp=cfg.k_tsp)
    parity.assert_scores_close(g["tsp"], res.T, what="tsp")
    parity.assert_selection_matches(g["idx_tsp"], res.idx_tsp, res.pooled_tsp, cfg.N, cfg.w, cfg.k_tsp)
    assert abs(g["tsp"].sum() - cfg.w * cfg.H) < 1e-3 * cfg.w * cfg.H


def test_cross_layer_accumulation():
    cfg = workloads.shrink(workloads.C5, N=3000, layers=3, k_kv=256, k_tsp=450, n_hitters=16)
    C = torch.zeros((cfg.Hkv, cfg.N), dtype=torch.float32, device="cuda")
    Cref = np.zeros((cfg.Hkv, cfg.N))
    for ell in range(1, cfg.layers + 1):
        lay = workloads.make_layer(cfg, layer=ell)
        kvc.kvc_score(dev_bf16(lay.q), dev_bf16(lay.k), accum=C)
        Cref += oracle.get().window_scores(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale)
    parity.assert_scores_close(C.cpu().numpy(), Cref, what="C_global")


# --------------------------------------------------------------------------- #
# ragged batch
# --------------------------------------------------------------------------- #
def test_varlen_matches_oracle_and_single_sequence_calls():
    cfg = workloads.shrink(workloads.C4, len_range=(200, 5000), k_kv=150, n_hitters=4, seed=4001)
    lay = workloads.make_layer(cfg)
    B = lay.batch
    lens = lay.lengths()
    cu = torch.from_numpy(lay.cu_seqlens).cuda()
    q = dev_bf16(lay.q).view(B, cfg.w, cfg.H, cfg.d)
    kd = dev_bf16(lay.k)
    vd = dev_bf16(lay.v)
    err = _err_word()
    scores = kvc.kvc_score_varlen(q, kd, cu, int(lens.max()), dev_err=err)
    idx, counts = kvc.kvc_select_topk_varlen(scores, cu, int(lens.max()), cfg.w, cfg.pool, cfg.k_kv, dev_err=err)
    ko, vo = kvc.kvc_gather_kv_varlen(kd, vd, cu, idx, dev_err=err)
    assert err.item() == 0
    S = scores.cpu().numpy()
    I = idx.cpu().numpy()
    KO = host_bits(ko)
    assert np.array_equal(counts.cpu().numpy(), np.minimum(cfg.k_kv, lens))
    orc = oracle.get()
    for b in range(B):
        s0, s1 = lay.cu_seqlens[b], lay.cu_seqlens[b + 1]
        qb, kb = lay.q[b * cfg.w:(b + 1) * cfg.w], lay.k[s0:s1]
        res = oracle.layer(qb, kb, cfg.H, cfg.Hkv, cfg.w, cfg.scale, cfg.pool, cfg.k_kv)
        parity.assert_scores_close(S[:, s0:s1], res.A, what=f"seq {b}")
        m = min(cfg.k_kv, lens[b])
        for g in range(cfg.Hkv):
            parity.assert_selection_matches(I[b, g, :m], res.idx_kv[g], res.pooled[g], lens[b], cfg.w, cfg.k_kv)
            assert np.all(I[b, g, m:] == -1)
        ref_k, _ = orc.gather_kv(kb, I[b, :, :m])
        assert np.array_equal(KO[b, :, :m], ref_k)
        assert np.all(KO[b, :, m:] == 0)
        # the same sequence through the single-sequence entry point: the key
        # chunking differs with the batch, so agreement is to rounding only
        s_single = kvc.kvc_score(dev_bf16(qb), dev_bf16(kb))
        parity.assert_scores_close(s_single.cpu().numpy(), S[:, s0:s1], rtol=2e-6, what=f"single vs varlen {b}")


def test_varlen_bad_seqlens_flagged():
    cfg = workloads.shrink(workloads.C4, len_range=(100, 300), batch=3, n_hitters=2)
    lay = workloads.make_layer(cfg)
    cu_np = lay.cu_seqlens.copy()
    cu_np[2] = cu_np[1] + 10  # sequence 1 shorter than the window
    cu = torch.from_numpy(cu_np).cuda()
    q = dev_bf16(lay.q).view(3, cfg.w, cfg.H, cfg.d)
    err = _err_word()
    scores = kvc.kvc_score_varlen(q, dev_bf16(lay.k), cu, 400, dev_err=err)
    idx, counts = kvc.kvc_select_topk_varlen(scores, cu, 400, cfg.w, cfg.pool, 64, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() & kvc.KVC_DEV_ERR_SEQLENS
    assert counts[1].item() == 0 and torch.all(idx[1] == -1)


def test_varlen_seqlens_past_the_total_flagged():
    """A cu_seqlens whose last sequence ends past the packed total: the
    selection and the K/V gather report KVC_DEV_ERR_SEQLENS and pad that
    sequence (-1 indices, zero rows) instead of reading past the buffers.  The
    buffers carry slack past the total, so that even an unguarded read would
    stay inside them."""
    rng = np.random.default_rng(12)
    lens = np.array([300, 400])
    total, slack = int(lens.sum()), 256
    scores = torch.from_numpy(rng.random((2, total + slack)).astype(np.float32)).cuda()[:, :total]
    cu_np = np.array([0, 300, total + 100], dtype=np.int32)  # sequence 1 runs 100 tokens past the total
    cu = torch.from_numpy(cu_np).cuda()
    err = _err_word()
    idx, counts = kvc.kvc_select_topk_varlen(scores, cu, 800, 16, 3, 64, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() & kvc.KVC_DEV_ERR_SEQLENS
    assert counts.cpu().tolist() == [64, 0]
    assert torch.all(idx[1] == -1)
    orc = oracle.get()
    S0 = scores[:, :300].cpu().numpy().astype(np.float64)
    for r in range(2):
        Sp = orc.rank_scores(S0[r], 300, 16, 3)
        parity.assert_selection_matches(idx[0, r].cpu().numpy(), orc.select_topk(Sp, 300, 16, 64), Sp, 300, 16,
                                        64)

    kbig = torch.from_numpy(rng.standard_normal((total + slack, 2, 64)).astype(np.float32)).to(torch.bfloat16)
    k = kbig.cuda()[:total]
    gidx = torch.from_numpy(rng.integers(0, 300, size=(2, 2, 16)).astype(np.int32)).cuda()
    err = _err_word()
    ko, _ = kvc.kvc_gather_kv_varlen(k, None, cu, gidx, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == kvc.KVC_DEV_ERR_SEQLENS  # the sequence bit only: no index is out of its range
    KO, K = host_bits(ko), host_bits(k)
    G = gidx.cpu().numpy()
    for g in range(2):
        assert np.array_equal(KO[0, g], K[G[0, g], g, :])
    assert not KO[1].any()


# --------------------------------------------------------------------------- #
# one layer split by KV head (the ranks emulated one after another)
# --------------------------------------------------------------------------- #
def test_kv_head_split_reproduces_the_layer():
    """Two ranks of a KV-head split run one after another on this GPU (no
    rank waits for another): each scores its four KV heads through strided
    views of the layer's tensors; their partial all-head rows are added (the
    all-reduce of a multi-GPU run); each then ranks the summed row and
    gathers its half of the hidden columns and its heads' K/V.  Against the
    oracle: TSP and K/V sets under the band rule, gathers bit-exact."""
    from long_context_kv_window_b200 import shard
    cfg = workloads.shrink(workloads.C3, N=20000, k_kv=2000, k_tsp=4000, hidden=1024, n_hitters=64, seed=88)
    lay = workloads.make_layer(cfg)
    q, k, v, x = (dev_bf16(a) for a in (lay.q, lay.k, lay.v, lay.x))
    parts = [shard.HeadSplitLayer(r, 2, cfg.N, cfg.H, cfg.Hkv, cfg.d, cfg.w, cfg.k_kv, cfg.k_tsp, cfg.hidden, "cuda",
                                  pool_kernel=cfg.pool) for r in range(2)]
    rows = [p.score_local(q, k) for p in parts]
    total = rows[0] + rows[1]
    for p in parts:
        p.tsp.copy_(total)
        p.finish(k, v, x)
    torch.cuda.synchronize()
    res = oracle.layer(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale, cfg.pool, cfg.k_kv, cfg.k_tsp)
    it = parts[0].idx_tsp[0].cpu().numpy()
    assert np.array_equal(it, parts[1].idx_tsp[0].cpu().numpy())
    parity.assert_selection_matches(it, res.idx_tsp, res.pooled_tsp, cfg.N, cfg.w, cfg.k_tsp, what="split TSP set")
    xc = np.concatenate([host_bits(p.x_c) for p in parts], axis=1)
    assert np.array_equal(xc, lay.x[it])
    for p in parts:
        assert p.dev_err.item() == 0
        parity.assert_scores_close(p.scores.cpu().numpy(), res.A[p.g0:p.g1], what=f"rank {p.rank} scores")
        idx = p.idx_kv.cpu().numpy()
        kc, vc = host_bits(p.k_c), host_bits(p.v_c)
        for gl, g in enumerate(range(p.g0, p.g1)):
            parity.assert_selection_matches(idx[gl], res.idx_kv[g], res.pooled[g], cfg.N, cfg.w, cfg.k_kv,
                                            what=f"split K/V set of head {g}")
            assert np.array_equal(kc[gl], lay.k[idx[gl], g, :]) and np.array_equal(vc[gl], lay.v[idx[gl], g, :])


# --------------------------------------------------------------------------- #
# decode attention over the compacted cache
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("H,Hkv,d,kk", [(32, 8, 128, 13107), (32, 8, 128, 1), (32, 8, 128, 63), (8, 8, 64, 64),
                                        (40, 8, 128, 4096), (16, 1, 128, 2000), (8, 2, 64, 65), (6, 3, 128, 777),
                                        (64, 8, 128, 300), (8, 8, 128, 2305)])
def test_decode_attention_matches_oracle(H, Hkv, d, kk):
    """One decode query per head over [Hkv][kk][d] retained entries: the
    128K layer's 13107 entries per head, single and ragged tiles, G = 1, 2,
    4, 5, 8 (the tensor-core kernel) and 16 query heads per KV head and
    head_dim 64 (the CUDA-core kernel); a few planted entries carry most of
    the attention, so the running reference of a warp jumps mid-chunk."""
    rng = np.random.default_rng(H * 1000 + kk + d)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((H, d)).astype(np.float32))
    kc = workloads.f32_to_bf16_bits(rng.standard_normal((Hkv, kk, d)).astype(np.float32))
    vc = workloads.f32_to_bf16_bits(rng.standard_normal((Hkv, kk, d)).astype(np.float32))
    if kk > 8:  # planted heavy entries: K aligned with the group's queries
        G = H // Hkv
        qf = workloads.bf16_bits_to_f32(q).reshape(Hkv, G, d).mean(axis=1)
        for g in range(Hkv):
            pos = rng.choice(kk, size=3, replace=False)
            u = qf[g] / np.linalg.norm(qf[g])
            kc[g, pos] = workloads.f32_to_bf16_bits((3.0 * np.sqrt(d) * u)[None, :].repeat(3, 0).astype(np.float32))
    err = _err_word()
    out = kvc.kvc_decode_attention(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.get().decode_attention(q, kc, vc, H, Hkv, 1 / math.sqrt(d))
    parity.assert_decode_close(out.cpu().numpy(), ref, what=f"decode H={H} Hkv={Hkv} d={d} kk={kk}")


def test_decode_workspace_reused_across_calls():
    """The tensor-core decode keeps one ticket counter per KV head in its
    workspace and returns it to zero: consecutive calls on one zero-filled
    workspace -- different queries, then a smaller cache with fewer chunks --
    all match the oracle."""
    rng = np.random.default_rng(77)
    H, Hkv, d = 32, 8, 128
    kc = workloads.f32_to_bf16_bits(rng.standard_normal((Hkv, 5000, d)).astype(np.float32))
    vc = workloads.f32_to_bf16_bits(rng.standard_normal((Hkv, 5000, d)).astype(np.float32))
    ws = torch.zeros(kvc.decode_workspace_size(H, Hkv, d, 5000), dtype=torch.uint8, device="cuda")
    orc = oracle.get()
    for call, kk in enumerate([5000, 5000, 5000, 700]):
        q = workloads.f32_to_bf16_bits(rng.standard_normal((H, d)).astype(np.float32))
        kcc, vcc = np.ascontiguousarray(kc[:, :kk]), np.ascontiguousarray(vc[:, :kk])
        out = kvc.kvc_decode_attention(dev_bf16(q), dev_bf16(kcc), dev_bf16(vcc), ws=ws)
        torch.cuda.synchronize()
        ref = orc.decode_attention(q, kcc, vcc, H, Hkv, 1 / math.sqrt(d))
        parity.assert_decode_close(out.cpu().numpy(), ref, what=f"call {call} (kk={kk}) on a reused workspace")
    assert int(ws[:Hkv * 4].view(torch.int32).abs().sum().item()) == 0, "ticket counters not returned to zero"


def test_decode_over_the_layers_compacted_cache():
    """The cache a 32K layer's K/V retention leaves (scores -> per-KV-head
    top-k -> K/V gather) decoded with a fresh query per head, against the
    oracle's decode of the same cache."""
    cfg = workloads.shrink(workloads.C2, N=32768, seed=202)
    lay = workloads.make_layer(cfg)
    q, k, v = dev_bf16(lay.q), dev_bf16(lay.k), dev_bf16(lay.v)
    scores = kvc.kvc_score(q, k)
    idx = kvc.kvc_select_topk(scores, cfg.w, cfg.pool, cfg.k_kv)
    kc, vc = kvc.kvc_gather_kv(k, v, idx)
    rng = np.random.default_rng(5)
    qd = workloads.f32_to_bf16_bits(rng.standard_normal((cfg.H, cfg.d)).astype(np.float32))
    out = kvc.kvc_decode_attention(dev_bf16(qd), kc, vc)
    torch.cuda.synchronize()
    ref = oracle.get().decode_attention(qd, host_bits(kc), host_bits(vc), cfg.H, cfg.Hkv, cfg.scale)
    parity.assert_decode_close(out.cpu().numpy(), ref, what="decode over the compacted 32K layer")


# --------------------------------------------------------------------------- #
# causal prefill attention with the rows' log-sum-exp
# --------------------------------------------------------------------------- #
def _prefill_inputs(rng, N, H, Hkv, d=128, planted=0):
    q = rng.standard_normal((N, H, d)).astype(np.float32)
    k = rng.standard_normal((N, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((N, Hkv, d)).astype(np.float32)
    if planted:  # keys aligned with the queries of their group: logits far above the rest, mid-sequence
        G = H // Hkv
        for pos in rng.choice(N, size=min(planted, N), replace=False):
            for g in range(Hkv):
                u = q[min(N - 1, pos + 3), g * G].copy()
                k[pos, g] = 4.0 * u / np.linalg.norm(u) * np.sqrt(d)
    return tuple(workloads.f32_to_bf16_bits(a) for a in (q, k, v))


def assert_prefill_close(out, lse, ref_out, ref_lse, v_bits, H, Hkv, what):
    """Outputs within 6e-3 of max |v| of the KV head (the bf16 probabilities
    and the bf16 output each round by <= 2^-9: a convex combination of V rows
    whose weights move by <= 2^-8 relative, plus the output rounding); the
    log-sum-exp within 2e-5 of max(1, |lse|) (fp32 logits, fp64 sums)."""
    G = H // Hkv
    vmax = np.abs(workloads.bf16_bits_to_f32(v_bits)).max(axis=(0, 2))          # [Hkv]
    bound = 6e-3 * np.repeat(vmax, G)[None, :, None]
    err = np.abs(out - ref_out)
    assert np.all(err <= bound), f"{what}: output error {float((err / bound).max()):.2f} x the bound"
    lerr = np.abs(lse - ref_lse) / np.maximum(1.0, np.abs(ref_lse))
    assert lerr.max() <= 2e-5, f"{what}: log-sum-exp error {lerr.max():.2e}"


@pytest.mark.parametrize("N,H,Hkv,planted", [(1, 4, 2, 0), (100, 4, 1, 3), (128, 8, 2, 0), (129, 4, 4, 2),
                                             (300, 6, 3, 5), (700, 32, 8, 8), (1000, 4, 2, 0)])
def test_prefill_attention_matches_oracle(N, H, Hkv, planted):
    """Causal attention with grouped heads against the float64 oracle: single
    and ragged query blocks, G = 1, 2, 4; planted keys make some rows' maxima
    jump by far more than the reference slack mid-sequence (the output
    rescale in TMEM).  The log-sum-exp only mode (no output) gives the same
    log-sum-exp."""
    rng = np.random.default_rng(N * 7 + H + planted)
    q, k, v = _prefill_inputs(rng, N, H, Hkv, planted=planted)
    err = _err_word()
    out, lse = kvc.kvc_prefill_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_err=err)
    _, lse2 = kvc.kvc_prefill_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), want_out=False)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(lse, lse2)
    ref_out, ref_lse = oracle.get().prefill_attention(q, k, v, H, Hkv, 1 / math.sqrt(128))
    assert_prefill_close(out.float().cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, v, H, Hkv,
                         f"prefill N={N} H={H} Hkv={Hkv}")


def test_prefill_log_sum_exp_scores_the_window_in_one_read():
    """The TSP layer's chain with the prefill attention as the producer: its
    window rows' log-sum-exp handed to kvc_score_lse (one read of K) gives the
    two-pass scores within 1e-3 of the oracle and, ranked, the oracle's TSP and
    K/V sets under the near-tie rule."""
    cfg = workloads.shrink(workloads.C3, N=4096, k_kv=410, k_tsp=819, n_hitters=16, seed=64)
    rng = np.random.default_rng(64)
    N, H, Hkv, w = cfg.N, cfg.H, cfg.Hkv, cfg.w
    q, k, v = _prefill_inputs(rng, N, H, Hkv)
    qd, kd, vd = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    _, lse = kvc.kvc_prefill_attention(qd, kd, vd, want_out=False)
    S1 = kvc.kvc_score_lse(qd[N - w:], kd, lse[N - w:])
    S2 = kvc.kvc_score(qd[N - w:], kd)
    torch.cuda.synchronize()
    qw = np.ascontiguousarray(q[N - w:])
    res = oracle.layer(qw, k, H, Hkv, w, 1 / math.sqrt(128), cfg.pool, cfg.k_kv, k_tsp=cfg.k_tsp)
    parity.assert_scores_close(S1.cpu().numpy(), res.A, what="scores from the prefill log-sum-exp")
    parity.assert_scores_close(S2.cpu().numpy(), res.A, what="two-pass scores")
    # the layer plan with the same normalisers: the same scores and sets as the direct calls
    plan = kvc.LayerPlan(N, H, Hkv, 128, w, cfg.k_kv, cfg.k_tsp, None, False, "cuda", pool_kernel=cfg.pool)
    outp = plan.run(qd[N - w:], kd, lse=lse[N - w:])
    torch.cuda.synchronize()
    assert torch.equal(outp.scores, S1)
    ik = kvc.kvc_select_topk(S1, w, cfg.pool, cfg.k_kv).cpu().numpy()
    it = kvc.kvc_select_topk(S1, w, cfg.pool, cfg.k_tsp, row_group=Hkv).cpu().numpy()[0]
    for g in range(Hkv):
        parity.assert_selection_matches(ik[g], res.idx_kv[g], res.pooled[g], N, w, cfg.k_kv, what=f"K/V set {g}")
    parity.assert_selection_matches(it, res.idx_tsp, res.pooled_tsp, N, w, cfg.k_tsp, what="TSP set")
    assert np.array_equal(outp.idx_kv.cpu().numpy(), ik) and np.array_equal(outp.idx_tsp.cpu().numpy()[0], it)


def test_new_kernels_are_deterministic_under_repetition():
    """Repeated calls give bit-identical results: the decode's last-CTA merge
    (ticket counters), the residual-VQ candidate list and per-row atomic
    minimum, and the prefill's warp-local references and TMEM rescales
    depend on no arrival order."""
    rng = np.random.default_rng(97)
    H, Hkv, d, kk = 32, 8, 128, 3000
    q = dev_bf16(workloads.f32_to_bf16_bits(rng.standard_normal((H, d)).astype(np.float32)))
    kc = dev_bf16(workloads.f32_to_bf16_bits(rng.standard_normal((Hkv, kk, d)).astype(np.float32)))
    vc = dev_bf16(workloads.f32_to_bf16_bits(rng.standard_normal((Hkv, kk, d)).astype(np.float32)))
    ws = torch.zeros(kvc.decode_workspace_size(H, Hkv, d, kk), dtype=torch.uint8, device="cuda")
    ref = kvc.kvc_decode_attention(q, kc, vc, ws=ws).clone()
    for _ in range(20):
        assert torch.equal(kvc.kvc_decode_attention(q, kc, vc, ws=ws), ref)
    C = torch.from_numpy(workloads.make_codebooks(4, 256, d, seed=5)).cuda()
    rows = kc.view(-1, d)
    rc, _ = kvc.kvc_rvq_encode(rows, C)
    rc = rc.clone()
    for _ in range(10):
        assert torch.equal(kvc.kvc_rvq_encode(rows, C)[0], rc)
    qp, kp, vp = (dev_bf16(a) for a in _prefill_inputs(rng, 1500, 8, 2, planted=4))
    o0, l0 = kvc.kvc_prefill_attention(qp, kp, vp)
    o0, l0 = o0.clone(), l0.clone()
    for _ in range(10):
        o1, l1 = kvc.kvc_prefill_attention(qp, kp, vp)
        assert torch.equal(o1, o0) and torch.equal(l1, l0)
    torch.cuda.synchronize()


def test_prefill_over_the_propagated_tokens():
    """The later layers' attention over the TSP-propagated tokens: the query,
    key and value rows of the selected positions (gathered as hidden rows,
    ascending) attend causally among themselves, against the oracle on the
    same compacted rows."""
    rng = np.random.default_rng(71)
    N, H, Hkv = 2048, 8, 2
    q, k, v = _prefill_inputs(rng, N, H, Hkv)
    idx = np.sort(rng.choice(N, size=600, replace=False)).astype(np.int32)
    it = torch.from_numpy(idx).cuda()
    qc = kvc.kvc_gather_hidden(dev_bf16(q).view(N, H * 128), it).view(-1, H, 128)
    kc = kvc.kvc_gather_hidden(dev_bf16(k).view(N, Hkv * 128), it).view(-1, Hkv, 128)
    vc = kvc.kvc_gather_hidden(dev_bf16(v).view(N, Hkv * 128), it).view(-1, Hkv, 128)
    out, lse = kvc.kvc_prefill_attention(qc, kc, vc)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.get().prefill_attention(q[idx], k[idx], v[idx], H, Hkv, 1 / math.sqrt(128))
    assert_prefill_close(out.float().cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse, v[idx], H, Hkv,
                         "prefill over the propagated tokens")


# --------------------------------------------------------------------------- #
# residual vector quantisation
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("n,d,S,M", [(1000, 128, 4, 256), (129, 128, 2, 256), (300, 64, 3, 64), (77, 128, 1, 16),
                                     (5000, 128, 8, 128)])
def test_rvq_encode_matches_oracle(n, d, S, M):
    """Random rows against random codebooks (stage s at scale 2^-s): codes
    identical to the oracle outside the near-tie band, and the returned
    residual is the row minus its reconstruction."""
    rng = np.random.default_rng(n + d + S + M)
    x = workloads.f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32))
    C = workloads.make_codebooks(S, M, d, seed=n + M)
    xd, Cd = dev_bf16(x), torch.from_numpy(C).cuda()
    residual = torch.empty((n, d), dtype=torch.float32, device="cuda")
    err = _err_word()
    codes, _ = kvc.kvc_rvq_encode(xd, Cd, residual=residual, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref_codes, gap = oracle.get().rvq_encode(x, C)
    gc = codes.cpu().numpy()
    near = parity.check_rvq_codes(gc, ref_codes, gap, x, C, what=f"rvq n={n} d={d} S={S} M={M}")
    assert near <= max(2, n // 100), f"{near} rows decided inside the near-tie band"
    xf = workloads.bf16_bits_to_f32(x).astype(np.float64)
    rec = sum(C[s][gc[:, s]].astype(np.float64) for s in range(S))
    np.testing.assert_allclose(residual.cpu().numpy(), xf - rec, rtol=0, atol=1e-5)


def test_rvq_encode_strided_rows():
    """Rows read through a row stride that is not a multiple of 8 elements
    (the element-wise load path) give the same codes and residual as the
    same rows stored contiguously (the 16-byte load path)."""
    rng = np.random.default_rng(515)
    n, d, S, M = 333, 128, 3, 128
    x = workloads.f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32))
    C = torch.from_numpy(workloads.make_codebooks(S, M, d, seed=12)).cuda()
    wide = torch.zeros((n, d + 4), dtype=torch.bfloat16, device="cuda")
    wide[:, :d] = dev_bf16(x)
    strided = wide[:, :d]
    assert strided.stride(0) == d + 4
    r1 = torch.empty((n, d), dtype=torch.float32, device="cuda")
    r2 = torch.empty((n, d), dtype=torch.float32, device="cuda")
    c1, _ = kvc.kvc_rvq_encode(dev_bf16(x), C, residual=r1)
    c2, _ = kvc.kvc_rvq_encode(strided, C, residual=r2)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(r1, r2)


def test_rvq_encode_crowded_codebook():
    """A codebook of 256 near-copies of one vector puts every codeword inside
    the candidate band of every row (more candidates than the parallel
    re-scoring list holds): the per-warp re-scoring path decides, against the
    oracle under the near-tie rule; a second, ordinary stage follows."""
    rng = np.random.default_rng(616)
    n, d, M = 300, 128, 256
    x = workloads.f32_to_bf16_bits(rng.standard_normal((n, d)).astype(np.float32))
    base = rng.standard_normal(d)
    C0 = base[None, :] + 1e-3 * rng.standard_normal((M, d))
    C1 = 0.5 * rng.standard_normal((M, d))
    C = np.stack([C0, C1]).astype(np.float32)
    codes, _ = kvc.kvc_rvq_encode(dev_bf16(x), torch.from_numpy(C).cuda())
    torch.cuda.synchronize()
    ref_codes, gap = oracle.get().rvq_encode(x, C)
    parity.check_rvq_codes(codes.cpu().numpy(), ref_codes, gap, x, C, what="rvq, crowded codebook")


def test_rvq_encode_planted_codes_and_ties():
    """Rows built as one codeword per stage (codebooks of entries +-8^-s,
    exact in bf16) come back with exactly those codes and a zero residual;
    a duplicated codeword resolves to the lower index."""
    rng = np.random.default_rng(71)
    n, d, M, S = 700, 128, 64, 3
    C = np.stack([rng.choice([-1.0, 1.0], size=(M, d)) * 8.0 ** -s for s in range(S)]).astype(np.float32)
    C[0, 40] = C[0, 9]  # codeword 40 duplicates codeword 9
    planted = rng.integers(0, M, size=(n, S))
    planted[:, 0] = np.where(planted[:, 0] == 40, 9, planted[:, 0])
    xf = sum(C[s][planted[:, s]].astype(np.float64) for s in range(S))
    x = workloads.f32_to_bf16_bits(xf.astype(np.float32))
    assert np.array_equal(workloads.bf16_bits_to_f32(x).astype(np.float64), xf)
    residual = torch.empty((n, d), dtype=torch.float32, device="cuda")
    codes, _ = kvc.kvc_rvq_encode(dev_bf16(x), torch.from_numpy(C).cuda(), residual=residual)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), planted)
    assert not residual.cpu().numpy().any()


def test_rvq_encode_the_layers_compacted_cache():
    """The compacted K cache of a 32K layer ([8][2048][128] as 16384 rows),
    four stages of 256 codewords, against the oracle."""
    cfg = workloads.shrink(workloads.C2, N=32768, seed=303)
    lay = workloads.make_layer(cfg)
    q, k = dev_bf16(lay.q), dev_bf16(lay.k)
    idx = kvc.kvc_select_topk(kvc.kvc_score(q, k), cfg.w, cfg.pool, cfg.k_kv)
    kc, _ = kvc.kvc_gather_kv(k, None, idx)
    rows = kc.view(-1, cfg.d)
    C = workloads.make_codebooks(4, 256, cfg.d, seed=9)
    codes, _ = kvc.kvc_rvq_encode(rows, torch.from_numpy(C).cuda())
    torch.cuda.synchronize()
    xb = host_bits(rows)
    ref_codes, gap = oracle.get().rvq_encode(xb, C)
    near = parity.check_rvq_codes(codes.cpu().numpy(), ref_codes, gap, xb, C, what="rvq of the compacted cache")
    assert near <= rows.shape[0] // 100


# --------------------------------------------------------------------------- #
# statistics
# --------------------------------------------------------------------------- #
def test_layer_stats_against_oracle():
    cfg = workloads.shrink(workloads.C5, N=6000, layers=1, k_tsp=None)
    lay = workloads.make_layer(cfg, layer=1)
    A = oracle.get().window_scores(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale)
    gpu_scores = kvc.kvc_score(dev_bf16(lay.q), dev_bf16(lay.k))
    st = kvc.kvc_layer_stats(gpu_scores, cfg.w * cfg.G).cpu().numpy()
    for g in range(cfg.Hkv):
        ref = oracle.get().layer_stats(A[g], cfg.w * cfg.G)
        parity.assert_scores_close(st[g], ref, what=f"stats head {g}")


def test_layer_stats_closed_forms():
    n = 5000
    uni = torch.full((1, n), 3.0, device="cuda")
    st = kvc.kvc_layer_stats(uni, 3.0 * n).cpu().numpy()[0]
    assert abs(st[0] - math.log(n)) < 1e-4 * math.log(n)
    assert abs(st[1] - 50 / n) < 1e-6 and abs(st[2]) < 1e-12
    one = torch.zeros((1, n), device="cuda")
    one[0, 17] = 2.0
    st = kvc.kvc_layer_stats(one, 2.0).cpu().numpy()[0]
    assert abs(st[0]) < 1e-7 and abs(st[1] - 1) < 1e-6 and abs(st[2] - (1 / n) * (1 - 1 / n)) < 1e-9


def test_varlen_select_rejects_sequences_longer_than_max_seqlen():
    """A max_seqlen below a real length must not overflow the kernel's shared
    memory: that sequence is reported and left unranked, the others are fine."""
    rng = np.random.default_rng(9)
    lens = np.array([300, 1200, 500])
    cu_np = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    scores = torch.from_numpy(rng.random((2, int(cu_np[-1]))).astype(np.float32)).cuda()
    err = _err_word()
    idx, counts = kvc.kvc_select_topk_varlen(scores, torch.from_numpy(cu_np).cuda(), 600, 16, 3, 100,
                                             dev_err=err)
    torch.cuda.synchronize()
    assert err.item() & kvc.KVC_DEV_ERR_SEQLENS
    c = counts.cpu().numpy()
    assert c.tolist() == [100, 0, 100]
    assert torch.all(idx[1] == -1)
    orc = oracle.get()
    S = scores.cpu().numpy().astype(np.float64)
    for b in (0, 2):
        for r in range(2):
            Sp = orc.rank_scores(S[r, cu_np[b]:cu_np[b + 1]], lens[b], 16, 3)
            ref = orc.select_topk(Sp, lens[b], 16, 100)
            parity.assert_selection_matches(idx[b, r].cpu().numpy(), ref, Sp, lens[b], 16, 100)


def test_layer_plan_matches_the_single_calls():
    """LayerPlan ranks the TSP set either by summing the KV-head score rows
    inside the selection or on the head-sum row that scoring writes
    (tsp_row=True); both sum the heads in the same order and precision, so
    the index sets are identical.  The K/V chain runs on a side stream; its
    results equal the direct calls."""
    cfg = workloads.shrink(workloads.C3, N=20000, k_kv=2000, k_tsp=4000, hidden=512)
    lay = workloads.make_layer(cfg)
    q, kd, vd, xd = dev_bf16(lay.q), dev_bf16(lay.k), dev_bf16(lay.v), dev_bf16(lay.x)
    plan = kvc.LayerPlan(cfg.N, cfg.H, cfg.Hkv, cfg.d, cfg.w, cfg.k_kv, cfg.k_tsp, cfg.hidden, True, "cuda",
                         pool_kernel=cfg.pool)
    out = plan.run(q, kd, vd, xd)
    plan_row = kvc.LayerPlan(cfg.N, cfg.H, cfg.Hkv, cfg.d, cfg.w, cfg.k_kv, cfg.k_tsp, cfg.hidden, True, "cuda",
                             pool_kernel=cfg.pool, tsp_row=True)
    out_row = plan_row.run(q, kd, vd, xd)
    torch.cuda.synchronize()
    assert out.tsp is None
    scores = kvc.kvc_score(q, kd)
    assert torch.equal(out.scores, scores)
    assert torch.equal(out_row.scores, scores)
    ref_tsp = scores[0].clone()
    for g in range(1, cfg.Hkv):
        ref_tsp += scores[g]
    assert torch.equal(out_row.tsp[0], ref_tsp)
    it = kvc.kvc_select_topk(scores, cfg.w, cfg.pool, cfg.k_tsp, row_group=cfg.Hkv)
    assert torch.equal(out.idx_tsp, it)
    assert torch.equal(out_row.idx_tsp, it)
    assert torch.equal(out_row.x_c, out.x_c)
    ik = kvc.kvc_select_topk(scores, cfg.w, cfg.pool, cfg.k_kv)
    assert torch.equal(out.idx_kv, ik)
    ko, vo = kvc.kvc_gather_kv(kd, vd, ik)
    assert torch.equal(out.k_c, ko) and torch.equal(out.v_c, vo)
    assert torch.equal(out.x_c, kvc.kvc_gather_hidden(xd, it.view(-1)))
    assert plan.dev_err.item() == 0


@pytest.mark.parametrize("sigma,pool,k", [(3.0, 7, 13107), (1.0, 7, 26214), (3.0, 1, 4000)])
def test_select_heavy_tailed_rows(sigma, pool, k):
    """Log-normal rows: a long upper tail stretches the sampled key window, so
    the threshold bin holds hundreds of keys and the kernel narrows them with
    histogram levels before ranking the survivors."""
    n, w, rows = 131072, 32, 4
    rng = np.random.default_rng(int(sigma * 10) + pool + k)
    S = np.exp(sigma * rng.standard_normal((rows, n))).astype(np.float32)
    idx = kvc.kvc_select_topk(torch.from_numpy(S).cuda(), w, pool, k).cpu().numpy()
    orc = oracle.get()
    for r in range(rows):
        Sp = orc.rank_scores(S[r].astype(np.float64), n, w, pool)
        parity.assert_selection_matches(idx[r], orc.select_topk(Sp, n, w, k), Sp, n, w, k)


def test_shared_accumulator_buffers_repeated_calls_stable():
    """40 query heads over 8 KV heads: 160 window rows per KV head need two
    TMEM accumulator buffers shared by four epilogue groups.  Many calls at a
    size with dozens of tiles per CTA: no bounded wait may time out and every
    call must give bit-identical scores (a warp reading a buffer before it
    was refilled would show up as a difference)."""
    cfg = workloads.shrink(workloads.C5, N=65536, layers=1)
    lay = workloads.make_layer(cfg)
    q, kd = dev_bf16(lay.q), dev_bf16(lay.k)
    err = _err_word()
    ref = kvc.kvc_score(q, kd, dev_err=err).clone()
    tsp = torch.empty(1, cfg.N, device="cuda")
    for _ in range(24):
        s = kvc.kvc_score(q, kd, tsp=tsp, dev_err=err)
        assert torch.equal(s, ref)
    torch.cuda.synchronize()
    assert err.item() == 0


# --------------------------------------------------------------------------- #
# one-pass scoring with the window rows' log-sum-exp given
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("base,N,H,Hkv,w", [("C2", 5000, 32, 8, 32), ("C2", 3000, 40, 8, 32), ("C1", 1500, 8, 2, 8)])
def test_score_with_given_log_sum_exp(base, N, H, Hkv, w):
    """kvc_score_lse against the oracle given the same fp32 normalisers,
    passed as a prefill attention lays them out ([H][n], viewed at the window
    columns), and against the two-pass kvc_score; the head-sum row too."""
    cfg = workloads.shrink(getattr(workloads, base), N=N, H=H, Hkv=Hkv, w=w, n_sinks=4, n_hitters=8,
                           seed=6000 + N)
    lay = workloads.make_layer(cfg, with_x=False)
    lse = oracle_pins.logsumexp_rows(lay.q, lay.k, H, Hkv, w, cfg.scale)      # float64 [w][H]
    full = np.zeros((H, N), dtype=np.float32)
    full[:, N - w:] = lse.T
    lse_dev = torch.from_numpy(full).cuda()[:, N - w:].t()                   # [w][H], strides (1, N)
    q, kd = dev_bf16(lay.q), dev_bf16(lay.k)
    err = _err_word()
    tsp = torch.empty(N, dtype=torch.float32, device="cuda")
    got = kvc.kvc_score_lse(q, kd, lse_dev, tsp=tsp, dev_err=err)
    two = kvc.kvc_score(q, kd, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle.get().window_scores_lse(lay.q, lay.k, full[:, N - w:].T.astype(np.float64), H, Hkv, w, cfg.scale)
    parity.assert_scores_close(got.cpu().numpy(), ref, what="given-lse scores")
    parity.assert_scores_close(tsp.cpu().numpy(), ref.sum(axis=0), what="given-lse head-sum row")
    parity.assert_scores_close(got.cpu().numpy(), two.cpu().numpy().astype(np.float64), what="one pass vs two")


# --------------------------------------------------------------------------- #
# dynamic pivot detection
# --------------------------------------------------------------------------- #
def _device_pivot(st_np, tau, l_min, l_max):
    stats = torch.from_numpy(np.ascontiguousarray(st_np, dtype=np.float32)).cuda()
    state = kvc.pivot_state("cuda")
    err = _err_word()
    for layer in range(1, st_np.shape[0] + 1):
        kvc.kvc_pivot_update(stats[layer - 1], layer, tau, l_min, l_max, state, dev_err=err)
    torch.cuda.synchronize()
    return kvc.pivot_layer(state), err.item()


def test_pivot_update_matches_oracle():
    """The device rule, fed one layer at a time, decides exactly the oracle's
    pivot: random statistic sequences, the hand-worked sequences of the pins,
    and a phase change whose statistics come from kvc_layer_stats."""
    orc = oracle.get()
    rng = np.random.default_rng(31)
    for trial in range(200):
        L, heads = int(rng.integers(2, 17)), int(rng.integers(1, 9))
        E = np.cumsum(-rng.exponential(0.3, size=L)) + 8.0
        st = np.zeros((L, heads, 3), dtype=np.float32)
        st[:, :, 0] = E[:, None] + rng.normal(0, 0.2, size=(L, heads))
        st[:, :, 1] = rng.random((L, heads))
        st[:, :, 2] = rng.random((L, heads))
        tau = float(rng.choice([0.0, 0.02, 0.05, 0.1]))
        l_min = int(rng.integers(1, L + 1))
        l_max = int(rng.integers(l_min, L + 1))
        got, err = _device_pivot(st, tau, l_min, l_max)
        assert err == 0
        assert got == orc.pivot_layer(st, tau, l_min, l_max), f"trial {trial}"
    for E, S, tau, lo, hi, want in [([5, 5, 5, 3, 3, 3], [0.1, 0.1, 0.1, 0.2, 0.3, 0.4], 0.25, 1, 6, 4),
                                    ([4, 4, 4, 3, 2, 2], [0.1, 0.1, 0.1, 0.2, 0.3, 0.4], 0.25, 1, 6, 4),
                                    ([4, 4, 4, 3.0000002, 2, 2], [0.1, 0.1, 0.1, 0.2, 0.3, 0.4], 0.25, 1, 6, 5)]:
        st = oracle_pins._stats(E, S)
        assert _device_pivot(st, tau, lo, hi) == (want, 0)
    # a phase change at layer 7, statistics on the GPU
    N, heads, L = 4096, 4, 12
    st = np.zeros((L, heads, 3), dtype=np.float32)
    for layer in range(1, L + 1):
        A = oracle_pins._phase_change_scores(rng, N, heads, layer, 7).astype(np.float32)
        st[layer - 1] = kvc.kvc_layer_stats(torch.from_numpy(A).cuda(), 1.0).cpu().numpy()
    assert orc.pivot_layer(st, 0.1, 2, 10) == 7
    assert _device_pivot(st, 0.1, 2, 10) == (7, 0)


def test_pivot_update_out_of_order_is_flagged():
    stats = torch.rand((4, 3), device="cuda")
    state = kvc.pivot_state("cuda")
    err = _err_word()
    kvc.kvc_pivot_update(stats, 1, 0.1, 1, 8, state, dev_err=err)
    before = state.clone()
    kvc.kvc_pivot_update(stats, 3, 0.1, 1, 8, state, dev_err=err)
    torch.cuda.synchronize()
    assert err.item() == kvc.KVC_DEV_ERR_ORDER
    assert torch.equal(state, before)

