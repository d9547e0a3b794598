"""Parity at the full workload sizes, in the launch configuration the
benchmark times (BF16 storage, tensor-core kernels, the same chunking and
key-range splits): every call runs on the whole problem, and sampled outputs
are compared with the oracle one by one (only the sampled rows are copied to
the host).

  csa_prefill_32k   B=1, T=32768     compress, indexer top-k, sparse attention
  hca_prefill_128k  B=1, T=131072    compress, dense attention
  csa_decode_1m     B=64, T=2^20     indexer top-k over 262144 entries, sparse attention
  stack_4layer_128k one CSA and one HCA layer at B=2, T=131072
"""
import math

import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as O
from workloads import gen, get_config

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


def sample_rows(T, n, seed):
    r = np.random.default_rng(seed)
    rows = set(r.choice(T, n - 4, replace=False).tolist()) | {0, 3, T // 2, T - 1}
    return sorted(rows)


def check_attn(got, ref, max_abs=1e-2, mean_abs=1e-3):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    assert err.max() <= max_abs, f"max abs err {err.max():.3e}"
    assert err.mean() <= mean_abs, f"mean abs err {err.mean():.3e}"


def check_indexer_rows(sc_rows, idx_rows, qi_rows, w_rows, k_i, positions, m, k, Nc):
    """Per sampled row: scores within 1e-3 relative of the oracle's, selection
    bit-exact on the GPU's own FP32 scores; recall >= 99.9 % overall."""
    hits = tot = 0
    for r, t in enumerate(positions):
        nv = O.n_visible(t, m, Nc)
        ref_idx, ref_s = O.indexer_topk(qi_rows[r:r + 1], w_rows[r:r + 1], k_i, t, m, k)
        got_s = sc_rows[r, :nv]
        ref = ref_s[0, :nv]
        if nv:
            scale = np.maximum(np.abs(ref), np.sqrt(np.mean(ref * ref)))
            assert (np.abs(got_s - ref) <= 1e-3 * scale).all(), f"position {t}: scores off"
        same = O.topk_select(got_s, k) if nv else np.full(k, -1)
        np.testing.assert_array_equal(idx_rows[r], same)
        rr = ref_idx[0][ref_idx[0] >= 0]
        hits += len(set(idx_rows[r][idx_rows[r] >= 0].tolist()) & set(rr.tolist()))
        tot += len(rr)
    assert tot == 0 or hits >= 0.999 * tot, f"recall {hits / tot:.5f}"


def check_attn_rows(out_rows, q_rows, positions, entries, ckv_b, m, kv_b, kv_pos0, W, sink, R):
    refs = [O.attend_one(q_rows[r], t, entries[r], ckv_b, m, kv_b, kv_pos0, W, sink, R)[0]
            for r, t in enumerate(positions)]
    check_attn(out_rows, np.stack(refs))


def _inputs(kind, cfg, seed, unit=False):
    B, T, D = cfg.B, cfg.T, cfg.D
    m = cfg.m if kind == "csa" else cfg.m_hca
    g = gen._gen(seed, DEV)
    s = 1.0 if unit else 1.0 / math.sqrt(D)
    x = {"kv": gen._randn((B, T, D), g, DEV, s, torch.bfloat16),
         "gate": gen._randn((B, T, D), g, DEV, 1.0, torch.bfloat16),
         "q": gen._randn((B, T, cfg.H, D), g, DEV, s, torch.bfloat16),
         "sink": gen._randn((cfg.H,), g, DEV)}
    if kind == "csa":
        x["q_idx"] = gen._randn((B, T, cfg.H_I, cfg.D_I), g, DEV, 1.0 / math.sqrt(cfg.D_I), torch.bfloat16)
        x["w"] = gen._randn((B, T, cfg.H_I), g, DEV, 1.0 / math.sqrt(cfg.H_I))
        x["k_idx"] = gen._randn((B, T // m, cfg.D_I), g, DEV, 1.0 / math.sqrt(cfg.D_I), torch.bfloat16)
    return x, m


def _run_csa_layer(lcsa, cfg, seed, n_rows):
    B, T, Nc = cfg.B, cfg.T, cfg.T // cfg.m
    x, m = _inputs("csa", cfg, seed)
    ckv = lcsa.csa_compress(x["kv"], x["gate"], m)                    # BF16 cache, as in the bench
    idx, sc = lcsa.indexer_topk(x["q_idx"], x["w"], x["k_idx"], 0, m, cfg.k, return_scores=True)
    rows = {b: sample_rows(T, n_rows, seed + b) for b in range(B)}
    for b in range(B):
        r = rows[b]
        ref_c = O.csa_compress(np64(x["kv"][b]), np64(x["gate"][b]), m)
        np.testing.assert_allclose(np64(ckv[b]), ref_c, rtol=8e-3, atol=2e-4)
        check_indexer_rows(np64(sc[b, r]), idx[b, r].cpu().numpy(), np64(x["q_idx"][b, r]), np64(x["w"][b, r]),
                           np64(x["k_idx"][b]), r, m, cfg.k, Nc)
    del sc
    torch.cuda.empty_cache()
    entries = {b: [idx[b, i][idx[b, i] >= 0].cpu().numpy() for i in rows[b]] for b in range(B)}
    # spec-scale inputs through the whole pipeline, then unit-scale attention on the same selection
    out = lcsa.csa_sparse_attn(x["q"], ckv, idx, x["kv"], x["sink"], 0, 0, m, cfg.W, cfg.R)
    for b in range(B):
        check_attn_rows(np64(out[b, rows[b]]), np64(x["q"][b, rows[b]]), rows[b], entries[b], np64(ckv[b]), m,
                        np64(x["kv"][b]), 0, cfg.W, np64(x["sink"]), cfg.R)
    del out, x, ckv
    torch.cuda.empty_cache()
    xu = gen.make_attn_inputs(B, T, cfg.H, cfg.D, Nc, T, "bf16", seed=seed + 50, device=DEV, unit_scale=True)
    out = lcsa.csa_sparse_attn(xu["q"], xu["ckv"], idx, xu["kv"], xu["sink"], 0, 0, m, cfg.W, cfg.R)
    for b in range(B):
        check_attn_rows(np64(out[b, rows[b]]), np64(xu["q"][b, rows[b]]), rows[b], entries[b], np64(xu["ckv"][b]),
                        m, np64(xu["kv"][b]), 0, cfg.W, np64(xu["sink"]), cfg.R)
    del out, xu, idx
    torch.cuda.empty_cache()
    assert lcsa.get_device_status() == 0


def _run_hca_layer(lcsa, cfg, seed, n_rows):
    B, T = cfg.B, cfg.T
    for unit in (False, True):
        x, m = _inputs("hca", cfg, seed + (7 if unit else 0), unit=unit)
        ckv = lcsa.hca_compress(x["kv"], x["gate"], m)
        out = lcsa.hca_dense_attn(x["q"], ckv, x["kv"], x["sink"], 0, 0, m, cfg.W, cfg.R)
        for b in range(B):
            rows = sample_rows(T, n_rows, seed + b)
            ref_c = O.hca_compress(np64(x["kv"][b]), np64(x["gate"][b]), m)
            np.testing.assert_allclose(np64(ckv[b]), ref_c, rtol=8e-3, atol=2e-4 * (8 if unit else 1))
            entries = [np.arange(O.n_visible(t, m, T // m)) for t in rows]
            check_attn_rows(np64(out[b, rows]), np64(x["q"][b, rows]), rows, entries, np64(ckv[b]), m,
                            np64(x["kv"][b]), 0, cfg.W, np64(x["sink"]), cfg.R)
        del x, ckv, out
        torch.cuda.empty_cache()
    assert lcsa.get_device_status() == 0


def test_csa_prefill_32k_full(lcsa):
    _run_csa_layer(lcsa, get_config("csa_prefill_32k"), seed=1001, n_rows=24)


def test_hca_prefill_128k_full(lcsa):
    _run_hca_layer(lcsa, get_config("hca_prefill_128k"), seed=1101, n_rows=24)


def test_csa_decode_1m_full(lcsa):
    cfg = get_config("csa_decode_1m")
    B, T, Nc, m = cfg.B, cfg.T, cfg.T // cfg.m, cfg.m
    ix = gen.make_indexer_inputs(B, 1, Nc, cfg.H_I, cfg.D_I, "bf16", seed=1201, device=DEV,
                                 boost_frac=cfg.boost_frac)
    idx, sc = lcsa.indexer_topk(ix["q_idx"], ix["w"], ix["k_idx"], T, m, cfg.k, return_scores=True)
    g = gen._gen(1202, DEV)
    ckv = gen._randn((B, Nc, cfg.D), g, DEV, 1.0, torch.bfloat16)             # unit scale
    q = gen._randn((B, 1, cfg.H, cfg.D), g, DEV, 1.0, torch.bfloat16)
    kvw = gen._randn((B, cfg.W, cfg.D), g, DEV, 1.0, torch.bfloat16)
    sink = gen._randn((cfg.H,), g, DEV)
    out = lcsa.csa_sparse_attn(q, ckv, idx, kvw, sink, T, T - cfg.W + 1, m, cfg.W, cfg.R)
    for b in (0, 17, 63):
        check_indexer_rows(np64(sc[b]), idx[b].cpu().numpy(), np64(ix["q_idx"][b]), np64(ix["w"][b]),
                           np64(ix["k_idx"][b]), [T], m, cfg.k, Nc)
        sel = idx[b, 0][idx[b, 0] >= 0].cpu().numpy()
        check_attn_rows(np64(out[b]), np64(q[b]), [T], [sel], np64(ckv[b]), m, np64(kvw[b]), T - cfg.W + 1,
                        cfg.W, np64(sink), cfg.R)
    assert lcsa.get_device_status() == 0


def test_csa_decode_1m_fp4_indexer_full(lcsa):
    """FP4 QK path at the decode size: MXFP4 keys (bit-exact with the oracle's
    quantiser), scores within 1e-3 relative of the oracle's on the quantised
    values, selection bit-exact on the GPU's scores."""
    cfg = get_config("csa_decode_1m")
    B, T, Nc, m = cfg.B, cfg.T, cfg.T // cfg.m, cfg.m
    ix = gen.make_indexer_inputs(B, 1, Nc, cfg.H_I, cfg.D_I, "bf16", seed=1211, device=DEV,
                                 boost_frac=cfg.boost_frac)
    kc, ks = lcsa.quantize_mxfp4(ix["k_idx"])
    idx, sc = lcsa.indexer_topk_mxfp4(ix["q_idx"], ix["w"], kc, ks, T, m, cfg.k, return_scores=True)
    for b in (0, 63):
        rkc, rks = O.quantize_mxfp4(np64(ix["k_idx"][b]))
        np.testing.assert_array_equal(kc[b].cpu().numpy(), rkc)
        np.testing.assert_array_equal(ks[b].cpu().numpy(), rks)
        ref_idx, ref_s = O.indexer_topk_mxfp4(np64(ix["q_idx"][b]), np64(ix["w"][b]), rkc, rks, T, m, cfg.k)
        got_s, ref = np64(sc[b, 0]), ref_s[0]
        scale = np.maximum(np.abs(ref), np.sqrt(np.mean(ref * ref)))
        assert (np.abs(got_s - ref) <= 1e-3 * scale).all()
        got = idx[b, 0].cpu().numpy()
        np.testing.assert_array_equal(got, O.topk_select(got_s, cfg.k))
        assert len(set(got.tolist()) & set(ref_idx[0].tolist())) >= 0.999 * cfg.k
    assert lcsa.get_device_status() == 0


def test_grouped_out_proj_full(lcsa):
    """Grouped output projection over the stack's token count (2 x 131072
    tokens, 64 heads x 512, g=8, d_g=1024, d=4096), sampled rows against the
    oracle."""
    T, n_h, c, g, d_g, d = 2 * 131072, 64, 512, 8, 1024, 4096
    gg = torch.Generator(device=DEV).manual_seed(1501)
    o = torch.randn(T, n_h, c, device=DEV, generator=gg).to(torch.bfloat16)
    K = n_h // g * c
    w1 = (torch.randn(g, d_g, K, device=DEV, generator=gg) / K ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(d, g * d_g, device=DEV, generator=gg) / (g * d_g) ** 0.5).to(torch.bfloat16)
    y = lcsa.grouped_out_proj(o, w1, w2)
    rows = sample_rows(T, 24, 1502)
    ref = O.grouped_out_proj(np64(o[rows]), np64(w1), np64(w2))
    got = np64(y[rows])
    scale = np.sqrt(np.mean(ref * ref))
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 * scale + 8e-3 * np.abs(ref).max() and err.mean() <= 2e-3 * scale
    assert lcsa.get_device_status() == 0


def test_stack_layers_full(lcsa):
    cfg = get_config("stack_4layer_128k")
    _run_csa_layer(lcsa, cfg, seed=1301, n_rows=12)
    _run_hca_layer(lcsa, cfg, seed=1401, n_rows=12)
