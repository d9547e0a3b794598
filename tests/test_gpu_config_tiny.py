"""The tiny CSA + HCA layer run end to end through the library, on every row,
against the oracle run end to end on the same inputs.

Workload: FP32, seed 0, B=1, T=1024, 4 query heads of dim 64 (last 32 rotary),
one shared K=V head, indexer 2 heads x 32, CSA m=4 (window 8) with top-64,
HCA m'=128 (8 entries), sliding window 64, a sink logit per head; kv, gate
logits, q and indexer q/k drawn N(0,1)/sqrt(dim).  The unit-scale twin draws
kv and q from N(0,1), so that the logits spread over O(1) and the attention
tolerance bites.

Chain per layer kind:
  CSA  csa_compress -> indexer_topk -> csa_sparse_attn
  HCA  hca_compress -> hca_dense_attn
Checked element by element: entries within 2e-6 absolute, indexer scores
within 1e-3 x max(|s|, rms(row)), the selection bit-exact on the library's own
scores and >= 99.9 % of the oracle's, attention (and its log-sum-exp) within
max-abs 1e-2 / mean-abs 1e-3 of the oracle's chain."""
import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as O
from workloads import gen
from workloads.configs import get_config

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def lcsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_library
    return build_library()


def np64(t):
    return t.detach().double().cpu().numpy()


def run_tiny_layer(lcsa, cfg, x):
    """The library's chain on the tiny layer's inputs (all rows)."""
    ckv_c = lcsa.csa_compress(x["kv"], x["gate"], cfg.m)
    ckv_h = lcsa.hca_compress(x["kv"], x["gate"], cfg.m_hca)
    idx, sc = lcsa.indexer_topk(x["q_idx"], x["w"], x["k_idx"], 0, cfg.m, cfg.k, return_scores=True)
    o_c, lse_c = lcsa.csa_sparse_attn(x["q"], ckv_c, idx, x["kv"], x["sink"], 0, 0, cfg.m, cfg.W, cfg.R,
                                      return_lse=True)
    o_h, lse_h = lcsa.hca_dense_attn(x["q"], ckv_h, x["kv"], x["sink"], 0, 0, cfg.m_hca, cfg.W, cfg.R,
                                     return_lse=True)
    torch.cuda.synchronize()
    return {"ckv_c": ckv_c, "ckv_h": ckv_h, "idx": idx, "scores": sc, "o_c": o_c, "lse_c": lse_c,
            "o_h": o_h, "lse_h": lse_h}


def oracle_tiny_layer(cfg, x):
    """The oracle's chain on the same inputs (FP64, selection in FP32)."""
    kv, gate, sink = np64(x["kv"][0]), np64(x["gate"][0]), np64(x["sink"])
    ckv_c = O.csa_compress(kv, gate, cfg.m)
    ckv_h = O.hca_compress(kv, gate, cfg.m_hca)
    idx, sc = O.indexer_topk(np64(x["q_idx"][0]), np64(x["w"][0]), np64(x["k_idx"][0]), 0, cfg.m, cfg.k)
    q = np64(x["q"])
    kvb = np64(x["kv"])
    o_c, lse_c = O.csa_sparse_attn(q, ckv_c[None], idx[None], kvb, 0, 0, cfg.m, cfg.W, sink, cfg.R)
    o_h, lse_h = O.hca_dense_attn(q, ckv_h[None], kvb, 0, 0, cfg.m_hca, cfg.W, sink, cfg.R)
    return {"ckv_c": ckv_c, "ckv_h": ckv_h, "idx": idx, "scores": sc, "o_c": o_c, "lse_c": lse_c,
            "o_h": o_h, "lse_h": lse_h}


def _assert_attn(got, ref, what):
    err = np.abs(np.asarray(got, dtype=np.float64).reshape(ref.shape) - ref)
    assert err.max() <= 1e-2, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= 1e-3, f"{what}: mean abs err {err.mean():.3e}"


@pytest.mark.parametrize("unit_scale", [False, True], ids=["spec_scale", "unit_scale"])
def test_tiny_layer_end_to_end(lcsa, unit_scale):
    cfg = get_config("tiny")
    assert (cfg.dtype, cfg.seed, cfg.B, cfg.T, cfg.H, cfg.D, cfg.R, cfg.H_I, cfg.D_I) == \
        ("fp32", 0, 1, 1024, 4, 64, 32, 2, 32)
    assert (cfg.m, cfg.m_hca, cfg.k, cfg.W) == (4, 128, 64, 64)
    x = gen.make_layer_inputs(cfg, device=DEV, unit_scale=unit_scale)
    got = run_tiny_layer(lcsa, cfg, x)
    ref = oracle_tiny_layer(cfg, x)
    T, Nc = cfg.T, cfg.T // cfg.m

    # compression: CSA 256 entries, HCA 8 entries
    assert got["ckv_c"].shape == (1, Nc, cfg.D) and got["ckv_h"].shape == (1, T // cfg.m_hca, cfg.D)
    np.testing.assert_allclose(np64(got["ckv_c"][0]), ref["ckv_c"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(np64(got["ckv_h"][0]), ref["ckv_h"], rtol=0, atol=2e-6)

    # indexer scores on every visible column of every row
    sc = np64(got["scores"][0])
    nv = [O.n_visible(t, cfg.m, Nc) for t in range(T)]
    for t in range(T):
        n = nv[t]
        if n == 0:
            continue
        r = ref["scores"][t, :n]
        scale = np.maximum(np.abs(r), np.sqrt(np.mean(r * r)))
        assert (np.abs(sc[t, :n] - r) <= 1e-3 * scale).all(), f"row {t}: indexer scores off"

    # selection: bit-exact on the library's own scores, recall against the oracle's chain
    gidx = got["idx"][0].cpu().numpy()
    np.testing.assert_array_equal(gidx, O.topk_from_scores(sc, nv, cfg.k))
    hits = sum(len(set(g[g >= 0]) & set(r[r >= 0])) for g, r in zip(gidx, ref["idx"]))
    tot = int((ref["idx"] >= 0).sum())
    assert tot == sum(min(cfg.k, n) for n in nv)
    assert hits >= 0.999 * tot, f"recall {hits / tot:.5f}"

    # attention: every row of both layer kinds against the oracle's chain.  A
    # row whose selection differs from the oracle's is compared with the
    # oracle's attention over the library's selection instead (its entries
    # are still checked above).
    same = np.array([np.array_equal(g, r) for g, r in zip(gidx, ref["idx"])])
    o_ref, lse_ref = ref["o_c"].copy(), ref["lse_c"].copy()
    diff_rows = [(0, int(t)) for t in np.nonzero(~same)[0]]
    if diff_rows:
        o_d, l_d = O.csa_sparse_attn(np64(x["q"]), ref["ckv_c"][None], gidx[None], np64(x["kv"]), 0, 0, cfg.m,
                                     cfg.W, np64(x["sink"]), cfg.R, rows=diff_rows)
        for n, (_, t) in enumerate(diff_rows):
            o_ref[t], lse_ref[t] = o_d[n], l_d[n]        # oracle rows are (b, i) pairs, B = 1
    _assert_attn(np64(got["o_c"]), o_ref, "csa_sparse_attn")
    np.testing.assert_allclose(np64(got["lse_c"]).reshape(lse_ref.shape), lse_ref, atol=2e-3)
    _assert_attn(np64(got["o_h"]), ref["o_h"], "hca_dense_attn")
    np.testing.assert_allclose(np64(got["lse_h"]).reshape(ref["lse_h"].shape), ref["lse_h"], atol=2e-3)
    assert lcsa.get_device_status() == 0
