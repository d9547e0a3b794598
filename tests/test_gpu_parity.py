"""Parity of every library call with the CPU oracle on the same seeded inputs
(sizes that span several tiles plus ragged tails, and the edge cases)."""
import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as O
from workloads import gen

pytestmark = pytest.mark.gpu

ATT_MAX, ATT_MEAN = 1e-2, 1e-3        # attention tolerance (BF16 in, FP32 accumulate, unit scale)


@pytest.fixture(scope="module")
def lcsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_library
    return build_library()


DEV = "cuda"


def np64(t):
    return t.detach().double().cpu().numpy()


def assert_attn_close(got, ref, max_abs=ATT_MAX, mean_abs=ATT_MEAN):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    assert err.max() <= max_abs, f"max abs err {err.max():.3e}"
    assert err.mean() <= mean_abs, f"mean abs err {err.mean():.3e}"


# ------------------------------------------------------------------ compress
@pytest.mark.parametrize("dtype,D", [("fp32", 64), ("bf16", 512), ("bf16", 64)])
@pytest.mark.parametrize("kind,m", [("csa", 4), ("hca", 128), ("csa", 3), ("hca", 16)])
@pytest.mark.parametrize("per_channel", [True, False])
def test_compress_parity(lcsa, dtype, D, kind, m, per_channel):
    B, T = 2, 1037                                   # ragged: T % m != 0
    x = gen.make_compress_inputs(B, T, D, dtype, seed=21, device=DEV, gate_per_channel=per_channel)
    fn = lcsa.csa_compress if kind == "csa" else lcsa.hca_compress
    ofn = O.csa_compress if kind == "csa" else O.hca_compress
    out = fn(x["kv"], x["gate"], m, out_dtype=torch.float32)
    assert out.shape == (B, T // m, D)
    for b in range(B):
        ref = ofn(np64(x["kv"][b]), np64(x["gate"][b]), m)
        np.testing.assert_allclose(np64(out[b]), ref, rtol=0, atol=2e-6)


def test_compress_bf16_out_and_rmsnorm(lcsa):
    B, T, D = 1, 512, 512
    x = gen.make_compress_inputs(B, T, D, "bf16", seed=22, device=DEV)
    w = torch.randn(D, device=DEV, generator=torch.Generator(device=DEV).manual_seed(5))
    out = lcsa.csa_compress(x["kv"], x["gate"], 4, rms_weight=w, rms_eps=1e-6)
    assert out.dtype == torch.bfloat16
    ref = O.csa_compress(np64(x["kv"][0]), np64(x["gate"][0]), 4, rms_weight=np64(w), rms_eps=1e-6)
    np.testing.assert_allclose(np64(out[0]), ref, rtol=1e-2, atol=1e-2)


def test_compress_short_sequence(lcsa):
    x = gen.make_compress_inputs(1, 3, 512, "bf16", seed=23, device=DEV)
    assert lcsa.csa_compress(x["kv"], x["gate"], 4).shape == (1, 0, 512)


@pytest.mark.parametrize("dtype,per_channel,rms", [("bf16", True, False), ("fp32", False, True), ("bf16", False, True)])
def test_compress_entries_from_a_buffer(lcsa, dtype, per_channel, rms):
    """Incremental compression from a buffer of raw rows equals the entries of
    the whole-sequence compression (CSA and HCA windows)."""
    B, T, D = 2, 1000, 512
    x = gen.make_compress_inputs(B, T, D, dtype, seed=27, device=DEV, gate_per_channel=per_channel)
    w = torch.randn(D, device=DEV, generator=torch.Generator(device=DEV).manual_seed(9)) if rms else None
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for m, window in ((4, 8), (128, 128), (16, 16)):
        ref = np.stack([O.compress(np64(x["kv"][b]), np64(x["gate"][b]), m, window,
                                   None if w is None else np64(w)) for b in range(B)])
        Nc = T // m
        j0, n = Nc // 3, Nc - Nc // 3 - 1                   # a middle range of entries
        pos0 = max(0, (j0 + 1) * m - window)
        hi = (j0 + n) * m
        cache = torch.zeros((B, Nc, D), dtype=tdt, device=DEV)
        lcsa.compress_entries(x["kv"][:, pos0:hi].contiguous(), x["gate"][:, pos0:hi].contiguous(), pos0, m, window,
                              j0, n, cache, rms_weight=w)
        tol = dict(rtol=8e-3, atol=2e-4) if dtype == "bf16" else dict(rtol=1e-5, atol=2e-6)
        np.testing.assert_allclose(np64(cache[:, j0:j0 + n]), ref[:, j0:j0 + n], **tol)
        assert not cache[:, :j0].any() and not cache[:, j0 + n:].any()   # nothing else touched


def test_compress_entries_decode_append(lcsa):
    """Decode: after every arriving token, the entry that just completed is
    appended from the 128-row window ring (CSA m=4 window 8, HCA m'=128)."""
    B, T, D, W = 3, 1024, 512, 128
    x = gen.make_compress_inputs(B, T, D, "bf16", seed=28, device=DEV)
    caches = {(4, 8): torch.zeros((B, T // 4, D), dtype=torch.bfloat16, device=DEV),
              (128, 128): torch.zeros((B, T // 128, D), dtype=torch.bfloat16, device=DEV)}
    for t in range(W, T + 1):                               # t tokens have arrived
        ring_kv = x["kv"][:, t - W:t].contiguous()
        ring_g = x["gate"][:, t - W:t].contiguous()
        for (m, window), cache in caches.items():
            if t % m == 0:
                lcsa.compress_entries(ring_kv, ring_g, t - W, m, window, t // m - 1, 1, cache)
    for (m, window), cache in caches.items():
        first = (W + m - 1) // m - 1 if W % m else W // m - 1     # first entry appended from the ring
        ref = np.stack([O.compress(np64(x["kv"][b]), np64(x["gate"][b]), m, window) for b in range(B)])
        np.testing.assert_allclose(np64(cache[:, first:]), ref[:, first:], rtol=8e-3, atol=2e-4)
    assert lcsa.get_device_status() == 0


# ------------------------------------------------------------------ top-k
@pytest.mark.parametrize("n_cols,k,ties", [(64, 8, 0), (1000, 64, 4), (8191, 2048, 0), (8191, 2048, 16),
                                          (40000, 2048, 0), (5000, 1, 3), (300, 2048, 0),
                                          (32768, 2048, 0), (262144, 2048, 0),   # cached / uncached rows
                                          (40000, 2048, 1), (262144, 2048, 2),   # threshold bin > candidate list
                                          (32768, 2048, 16), (32768, 2048, 1),   # shared-memory kernel: ties,
                                          (4096, 2048, 0), (2052, 2048, 3)])     # bucket overflow, n just above k
def test_topk_bitexact(lcsa, n_cols, k, ties):
    rows = 37 if n_cols < 100000 else 6
    s = gen.make_scores(rows, n_cols, seed=31 + n_cols, device=DEV, tie_levels=ties)
    g = torch.Generator(device="cpu").manual_seed(7)
    nv = torch.randint(0, n_cols + 1, (rows,), generator=g, dtype=torch.int32)
    nv[0], nv[1] = n_cols, min(k, n_cols)
    idx = lcsa.topk_from_scores(s, k, n_valid=nv.to(DEV))
    ref = O.topk_from_scores(s.cpu().double().numpy(), nv.numpy(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_adversarial_rows(lcsa):
    k = 16
    rows = [np.zeros(100), np.full(100, -3.5), np.r_[np.full(50, 1.0), np.full(50, -0.0)],
            np.r_[np.full(30, -0.0), np.full(70, 0.0)], np.linspace(-1, 1, 100)[::-1].copy(),
            np.r_[np.full(99, -np.inf), [0.0]], np.r_[[np.inf], np.zeros(99)]]
    s = torch.tensor(np.stack(rows), dtype=torch.float32, device=DEV)
    idx = lcsa.topk_from_scores(s, k)
    ref = O.topk_from_scores(s.cpu().double().numpy(), [100] * len(rows), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


@pytest.mark.parametrize("n_cols,k,ties", [(262144, 2048, 0), (40000, 2048, 1), (70001, 64, 0), (50000, 6, 0)])
def test_topk_long_rows_both_paths(lcsa, n_cols, k, ties):
    """Rows longer than one shared-memory chunk: the two-phase path (chunk
    top-k, then top-k of their union) and the single-phase kernel agree with
    the oracle; k = 6 has no two-phase path."""
    rows = 5
    s = gen.make_scores(rows, n_cols, seed=41 + n_cols, device=DEV, tie_levels=ties)
    nv = torch.tensor([n_cols, k, n_cols // 2 + 3, 32768 + 5, 32767][:rows], dtype=torch.int32)
    ref = O.topk_from_scores(s.cpu().double().numpy(), nv.numpy(), k)
    for ws in (None, False):
        idx = lcsa.topk_from_scores(s, k, n_valid=nv.to(DEV), workspace=ws)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref)
    assert (lcsa.topk_workspace_bytes(rows, n_cols, k) > 0) == (k % 4 == 0)


@pytest.mark.parametrize("n_cols", [8000, 20000])
def test_topk_pivot_bucket_sizes(lcsa, n_cols):
    """Rows built so that the k-th score sits inside a tight cluster of c
    scores (one value bucket): c = 20, 150, 600 and 3000 reach the one-warp,
    one-thread-per-entry, radix and whole-row resolutions of that bucket; the
    second half of the rows repeats values inside the cluster (ties)."""
    k = 2048
    g = np.random.default_rng(11)
    rows = []
    for ties in (False, True):
        for c in (20, 150, 600, 3000):
            r = g.standard_normal(n_cols).astype(np.float32)
            above = k - c // 2                               # scores above the cluster
            pos = g.permutation(n_cols)
            r[pos[:above]] = 20.0 + g.random(above).astype(np.float32)
            jit = (np.arange(c) % 7 if ties else np.arange(c)).astype(np.float32) * np.float32(1e-6)
            r[pos[above:above + c]] = np.float32(10.0) + jit
            rows.append(r)
    s = torch.tensor(np.stack(rows), device=DEV)
    idx = lcsa.topk_from_scores(s, k)
    ref = O.topk_from_scores(s.cpu().double().numpy(), [n_cols] * len(rows), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_skewed_rows(lcsa):
    """Rows whose value range is dominated by outliers (one sampled bucket
    holds nearly everything), infinities and constant rows."""
    n, k = 6000, 2048
    g = np.random.default_rng(5)
    base = g.standard_normal((6, n)).astype(np.float32)
    base[0, 17] = 1e30                                    # one huge outlier
    base[1, ::7] = -1e30                                  # many huge negatives
    base[2, 100:110] = np.inf                             # +inf entries
    base[3, :] = 0.25                                     # constant row
    base[4, ::2] = -np.inf                                # half the row -inf
    base[5, :] = np.round(base[5, :] * 4) / 4             # coarse levels, ties everywhere
    s = torch.tensor(base, device=DEV)
    idx = lcsa.topk_from_scores(s, k)
    ref = O.topk_from_scores(s.cpu().double().numpy(), [n] * 6, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_topk_toy_from_pages(lcsa):
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "topk_toy.json")))
    s = torch.tensor([g["scores"]], dtype=torch.float32, device=DEV)
    assert lcsa.topk_from_scores(s, g["k"]).cpu().tolist() == [g["expected_idx"]]


# ------------------------------------------------------------------ indexer
def _score_err_ok(got, ref, nv):
    for i in range(ref.shape[0]):
        n = nv[i]
        if n == 0:
            continue
        r, g_ = ref[i, :n], got[i, :n]
        scale = np.maximum(np.abs(r), np.sqrt(np.mean(r * r)))
        bad = np.abs(g_ - r) > 1e-3 * scale
        assert not bad.any(), f"row {i}: {int(bad.sum())} scores off, worst {np.max(np.abs(g_ - r) / scale):.2e}"


@pytest.mark.parametrize("dtype,H_I,D_I,Tq,Nc,m,k,q_pos0", [
    ("fp32", 2, 32, 300, 256, 4, 64, 724),          # tiny-layer shapes, tail rows
    ("bf16", 64, 128, 260, 1030, 4, 256, 3900),     # layer shapes, several tiles + ragged tail
    ("bf16", 64, 128, 37, 700, 4, 2048, 0),         # N_vis < k everywhere
    ("bf16", 16, 64, 50, 333, 4, 32, 1200),         # other shape on the CUDA-core kernel
])
def test_indexer_scores_and_recall(lcsa, dtype, H_I, D_I, Tq, Nc, m, k, q_pos0):
    B = 2
    x = gen.make_indexer_inputs(B, Tq, Nc, H_I, D_I, dtype, seed=41, device=DEV)
    idx, sc = lcsa.indexer_topk(x["q_idx"], x["w"], x["k_idx"], q_pos0, m, k, return_scores=True)
    hits = tot = 0
    for b in range(B):
        ref_idx, ref_s = O.indexer_topk(np64(x["q_idx"][b]), np64(x["w"][b]), np64(x["k_idx"][b]), q_pos0, m, k)
        nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
        _score_err_ok(np64(sc[b]), ref_s, nv)
        got = idx[b].cpu().numpy()
        # structure: ascending valid prefix, -1 padding, all visible
        for i in range(Tq):
            v = got[i][got[i] >= 0]
            assert (np.diff(v) > 0).all() and (v < max(nv[i], 1)).all()
            assert len(v) == min(k, nv[i]) and (got[i][len(v):] == -1).all()
            hits += len(set(v) & set(ref_idx[i][ref_idx[i] >= 0]))
            tot += int((ref_idx[i] >= 0).sum())
        # same scores -> identical selection
        sel = O.topk_from_scores(np64(sc[b]), nv, k)
        np.testing.assert_array_equal(got, sel)
    assert hits >= 0.999 * tot, f"recall {hits / tot:.5f}"


# ------------------------------------------------------------------ FP4 (MXFP4) indexer path
def _mx_inputs(seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(37, 160, generator=g) * torch.exp2(torch.randint(-30, 30, (37, 1), generator=g).float())
    # round-to-nearest-even midpoints and saturation (amax 7 fixes X = 0)
    x[0, :32] = torch.tensor([7.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.75, -5.0, -0.25, 0.0] + [0.1] * 20)
    x[1, :32] = 0.0                                   # all-zero block
    x[1, 32:64] = -0.0
    x[2, :32] = 1e-40 * torch.arange(32)              # FP32 subnormals
    x[3, 64:96] = torch.linspace(-6, 6, 32) * 2.0 ** 100
    x[4, 96:128] = torch.linspace(-1, 1, 32) * 2.0 ** -126
    return x


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_quantize_mxfp4_bit_exact(lcsa, dtype):
    x = _mx_inputs(61)
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    codes, scales = lcsa.quantize_mxfp4(x.to(DEV))
    rc, rs = O.quantize_mxfp4(x.double().numpy())
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)


def test_quantize_mxfp4_nonfinite_blocks(lcsa):
    x = torch.randn(3, 96, generator=torch.Generator().manual_seed(62))
    x[0, 3] = float("nan")
    x[1, 40] = float("inf")
    x[2, 95] = -float("inf")
    codes, scales = lcsa.quantize_mxfp4(x.to(DEV))
    rc, rs = O.quantize_mxfp4(x.double().numpy())
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    assert rs[0, 0] == 255 and rs[1, 1] == 255 and rs[2, 2] == 255


@pytest.mark.parametrize("Tq,Nc,m,k,q_pos0", [
    (260, 1030, 4, 256, 3900),      # 4-row query groups, several tiles + ragged tail
    (37, 700, 4, 2048, 0),          # N_vis < k everywhere
    (1, 3000, 4, 512, 12000),       # decode: one row per sequence, entry-range splits
    (6, 2100, 4, 128, 8000),        # a 4-row and a 2-row group
    (3, 20000, 4, 2048, 80000),     # long rows: two-phase top-k
])
def test_indexer_mxfp4_scores_and_selection(lcsa, Tq, Nc, m, k, q_pos0):
    B = 2
    x = gen.make_indexer_inputs(B, Tq, Nc, 64, 128, "bf16", seed=43, device=DEV)
    kc, ks = lcsa.quantize_mxfp4(x["k_idx"])
    idx, sc = lcsa.indexer_topk_mxfp4(x["q_idx"], x["w"], kc, ks, q_pos0, m, k, return_scores=True)
    hits = tot = 0
    for b in range(B):
        rkc, rks = O.quantize_mxfp4(np64(x["k_idx"][b]))
        np.testing.assert_array_equal(kc[b].cpu().numpy(), rkc)
        np.testing.assert_array_equal(ks[b].cpu().numpy(), rks)
        ref_idx, ref_s = O.indexer_topk_mxfp4(np64(x["q_idx"][b]), np64(x["w"][b]), rkc, rks, q_pos0, m, k)
        nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
        _score_err_ok(np64(sc[b]), ref_s, nv)
        got = idx[b].cpu().numpy()
        for i in range(Tq):
            v = got[i][got[i] >= 0]
            assert (np.diff(v) > 0).all() and (v < max(nv[i], 1)).all()
            assert len(v) == min(k, nv[i]) and (got[i][len(v):] == -1).all()
            hits += len(set(v) & set(ref_idx[i][ref_idx[i] >= 0]))
            tot += int((ref_idx[i] >= 0).sum())
        np.testing.assert_array_equal(got, O.topk_from_scores(np64(sc[b]), nv, k))
    assert hits >= 0.999 * tot, f"recall {hits / tot:.5f}"


def test_indexer_mxfp4_wide_block_scales(lcsa):
    # entries whose blocks differ by up to 2^13 stay exact on the E4M3 staging;
    # one block 2^20 below its entry's largest rounds there, within tolerance
    B, Tq, Nc, m, k, q_pos0 = 1, 4, 300, 4, 64, 1400
    x = gen.make_indexer_inputs(B, Tq, Nc, 64, 128, "bf16", seed=44, device=DEV)
    kf = x["k_idx"].float()
    kf[0, :, 32:64] *= 2.0 ** -13
    kf[0, :, 64:96] *= 2.0 ** 6
    kf[0, 7, 96:128] *= 2.0 ** -20
    k_idx = kf.to(torch.bfloat16)
    kc, ks = lcsa.quantize_mxfp4(k_idx)
    idx, sc = lcsa.indexer_topk_mxfp4(x["q_idx"], x["w"], kc, ks, q_pos0, m, k, return_scores=True)
    rkc, rks = O.quantize_mxfp4(np64(k_idx[0]))
    ref_idx, ref_s = O.indexer_topk_mxfp4(np64(x["q_idx"][0]), np64(x["w"][0]), rkc, rks, q_pos0, m, k)
    nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    _score_err_ok(np64(sc[0]), ref_s, nv)
    np.testing.assert_array_equal(idx[0].cpu().numpy(), O.topk_from_scores(np64(sc[0]), nv, k))


def _mxfp4_direct(lcsa, *args, **kw):
    """The call with the block-scaled MMA on the E2M1 keys (mode 1), then back to the default."""
    try:
        lcsa.set_fp4_mma(1)
        return lcsa.indexer_topk_mxfp4(*args, **kw)
    finally:
        lcsa.set_fp4_mma(0)


def _mxfp4_both_paths(lcsa, x, kc, ks, q_pos0, m, k):
    """Scores and selection with the block-scaled MMA and with the E4M3 staging path (default)."""
    direct = _mxfp4_direct(lcsa, x["q_idx"], x["w"], kc, ks, q_pos0, m, k, return_scores=True)
    staged = lcsa.indexer_topk_mxfp4(x["q_idx"], x["w"], kc, ks, q_pos0, m, k, return_scores=True)
    assert lcsa.get_device_status() == 0
    return direct, staged


@pytest.mark.parametrize("B,Tq,Nc,q_pos0,k", [
    (2, 1, 3000, 12000, 512),       # decode: entry-range splits, ragged last tile
    (3, 2, 1030, 4100, 256),        # two rows per sequence, ragged tail
    (1, 1, 100, 400, 64),           # less than one tile
    (2, 1, 20000, 80000, 2048),     # long rows: the code and scale rings wrap many times
    (1, 2, 64, 40, 64),             # the second row sees one more entry than the first
])
def test_indexer_mxfp4_block_scaled_mma(lcsa, B, Tq, Nc, q_pos0, k):
    # one- and two-row calls read the E2M1 codes and their block scales on the
    # tensor cores: same scores as the oracle and as the E4M3 staging path
    m = 4
    x = gen.make_indexer_inputs(B, Tq, Nc, 64, 128, "bf16", seed=47, device=DEV)
    kc, ks = lcsa.quantize_mxfp4(x["k_idx"])
    assert kc.data_ptr() % 32 == 0
    (idx1, sc1), (idx0, sc0) = _mxfp4_both_paths(lcsa, x, kc, ks, q_pos0, m, k)
    for b in range(B):
        rkc, rks = O.quantize_mxfp4(np64(x["k_idx"][b]))
        _, ref_s = O.indexer_topk_mxfp4(np64(x["q_idx"][b]), np64(x["w"][b]), rkc, rks, q_pos0, m, k)
        nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
        _score_err_ok(np64(sc1[b]), ref_s, nv)
        np.testing.assert_array_equal(idx1[b].cpu().numpy(), O.topk_from_scores(np64(sc1[b]), nv, k))
        for i in range(Tq):
            n = nv[i]
            r, d = ref_s[i, :n], np64(sc1[b])[i, :n] - np64(sc0[b])[i, :n]
            # the same exact products summed in FP32 in another order
            assert (np.abs(d) <= 1e-5 * np.maximum(np.abs(r), np.sqrt(np.mean(r * r)))).all()


def test_indexer_mxfp4_block_scaled_wide_block_scales(lcsa):
    # blocks 2^-13, 2^6 and 2^-20 away from the others: the block-scaled path
    # keeps every product exact, the 2^-20 block included
    B, Tq, Nc, m, k, q_pos0 = 1, 2, 300, 4, 64, 1400
    x = gen.make_indexer_inputs(B, Tq, Nc, 64, 128, "bf16", seed=44, device=DEV)
    kf = x["k_idx"].float()
    kf[0, :, 32:64] *= 2.0 ** -13
    kf[0, :, 64:96] *= 2.0 ** 6
    kf[0, 7, 96:128] *= 2.0 ** -20
    k_idx = kf.to(torch.bfloat16)
    kc, ks = lcsa.quantize_mxfp4(k_idx)
    idx, sc = _mxfp4_direct(lcsa, x["q_idx"], x["w"], kc, ks, q_pos0, m, k, return_scores=True)
    rkc, rks = O.quantize_mxfp4(np64(k_idx[0]))
    _, ref_s = O.indexer_topk_mxfp4(np64(x["q_idx"][0]), np64(x["w"][0]), rkc, rks, q_pos0, m, k)
    nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    for i in range(Tq):
        r, g_ = ref_s[i, :nv[i]], np64(sc[0])[i, :nv[i]]
        assert (np.abs(g_ - r) <= 1e-5 * np.maximum(np.abs(r), np.sqrt(np.mean(r * r)))).all()
    np.testing.assert_array_equal(idx[0].cpu().numpy(), O.topk_from_scores(np64(sc[0]), nv, k))


def test_indexer_mxfp4_codes_16_byte_aligned_take_staging(lcsa):
    # codes 16 but not 32 bytes aligned: the call falls back to the staging
    # path and gives its results bit for bit
    B, Tq, Nc, m, k, q_pos0 = 2, 1, 900, 4, 128, 3600
    x = gen.make_indexer_inputs(B, Tq, Nc, 64, 128, "bf16", seed=48, device=DEV)
    kc, ks = lcsa.quantize_mxfp4(x["k_idx"])
    buf = torch.empty(B * Nc * 64 + 16, dtype=torch.uint8, device=DEV)
    kc16 = buf[16:].view(B, Nc, 64)
    kc16.copy_(kc)
    assert kc16.data_ptr() % 32 == 16
    got = _mxfp4_direct(lcsa, x["q_idx"], x["w"], kc16, ks, q_pos0, m, k, return_scores=True)
    (_, _), (idx0, sc0) = _mxfp4_both_paths(lcsa, x, kc, ks, q_pos0, m, k)
    nv = O.n_visible(q_pos0, m, Nc)
    assert torch.equal(got[0], idx0) and torch.equal(got[1][..., :nv], sc0[..., :nv])


def test_indexer_mxfp4_small_workspace_chunks(lcsa):
    B, Tq, Nc, m, k, q_pos0 = 2, 40, 900, 4, 128, 3600
    x = gen.make_indexer_inputs(B, Tq, Nc, 64, 128, "bf16", seed=45, device=DEV)
    kc, ks = lcsa.quantize_mxfp4(x["k_idx"])
    full = lcsa.indexer_topk_mxfp4(x["q_idx"], x["w"], kc, ks, q_pos0, m, k)
    need = lcsa.indexer_mxfp4_workspace_bytes(x["q_idx"], kc, k)
    small = torch.empty(need // 9, dtype=torch.uint8, device=DEV)     # a few rows at a time
    part = lcsa.indexer_topk_mxfp4(x["q_idx"], x["w"], kc, ks, q_pos0, m, k, workspace=small)
    assert torch.equal(full, part)


# ------------------------------------------------------------------ grouped output projection
@pytest.mark.parametrize("T,n_h,c,g,d_g,d", [
    (300, 64, 512, 8, 1024, 4096),     # layer shapes, ragged token count (3 m-tiles, tail of 44)
    (129, 64, 512, 4, 512, 1024),      # other grouping
    (64, 8, 64, 2, 224, 136),          # N not a multiple of the 256-column tile, small K
    (17, 64, 512, 1, 1024, 512),       # one group
])
def test_grouped_out_proj_parity(lcsa, T, n_h, c, g, d_g, d):
    gen_ = torch.Generator(device=DEV).manual_seed(71)
    o = torch.randn(T, n_h, c, device=DEV, generator=gen_).to(torch.bfloat16)
    K = n_h // g * c
    w1 = (torch.randn(g, d_g, K, device=DEV, generator=gen_) / K ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(d, g * d_g, device=DEV, generator=gen_) / (g * d_g) ** 0.5).to(torch.bfloat16)
    y = lcsa.grouped_out_proj(o, w1, w2)
    ref = O.grouped_out_proj(np64(o), np64(w1), np64(w2))
    got = np64(y)
    scale = np.sqrt(np.mean(ref * ref))
    err = np.abs(got - ref)
    # BF16 output (relative 2^-9) plus FP32 accumulation and BF16 intermediate rounding differences
    assert err.max() <= 2e-2 * scale + 8e-3 * np.abs(ref).max(), f"max err {err.max():.3e} (rms {scale:.3e})"
    assert err.mean() <= 2e-3 * scale, f"mean err {err.mean():.3e}"


# ------------------------------------------------------------------ attention
def _attn_case(B, Tq, H, D, Nc, Tkv, dtype, seed, unit=True, sink=True):
    return gen.make_attn_inputs(B, Tq, H, D, Nc, Tkv, dtype, seed=seed, device=DEV, unit_scale=unit,
                                with_sink=sink)


def _sink(x):
    return None if x["sink"] is None else np64(x["sink"])


@pytest.mark.parametrize("Tq,q_pos0,W", [(300, 0, 128), (77, 5000, 128), (40, 1000, 100)])
def test_sliding_window_only_layer(lcsa, Tq, q_pos0, W):
    """A pure sliding-window layer (the first two V4-Flash layers): the core
    attention with an empty entry cache, i.e. window + sink only."""
    B, H, D, R = 2, 64, 512, 64
    Tkv = q_pos0 + Tq
    x = _attn_case(B, Tq, H, D, 0, Tkv, "bf16", seed=55)
    assert x["ckv"].shape == (B, 0, D)
    out = lcsa.hca_dense_attn(x["q"], x["ckv"], x["kv"], x["sink"], q_pos0, 0, 128, W, R)
    ref, _ = O.hca_dense_attn(np64(x["q"]), np64(x["ckv"]), np64(x["kv"]), q_pos0, 0, 128, W, _sink(x), R)
    assert_attn_close(np64(out).reshape(ref.shape), ref)


@pytest.mark.parametrize("dtype,H,D,R,m,W,k,Tq,Nc,q_pos0,unit", [
    ("fp32", 4, 64, 32, 4, 64, 64, 200, 256, 824, True),       # tiny layer: rows near the end of T=1024
    ("fp32", 4, 64, 32, 4, 64, 64, 64, 256, 0, True),          # first rows: no entries / short window
    ("bf16", 64, 512, 64, 4, 128, 256, 40, 700, 2700, True),   # layer shapes
    ("bf16", 64, 512, 64, 4, 128, 256, 40, 700, 2700, False),  # spec scale
    ("bf16", 64, 512, 64, 4, 128, 2048, 9, 3000, 9000, True),  # full k
    ("bf16", 64, 512, 64, 4, 100, 100, 20, 900, 3000, True),   # odd W and k
    ("bf16", 64, 512, 64, 4, 128, 256, 160, 700, 2700, True),  # >= 296 rows: no key-range split
    ("bf16", 64, 512, 64, 4, 128, 3000, 4, 5000, 19000, True), # k > 2048: forced key-range splits
])
def test_csa_sparse_attn_parity(lcsa, dtype, H, D, R, m, W, k, Tq, Nc, q_pos0, unit):
    B = 2
    Tkv = q_pos0 + Tq
    x = _attn_case(B, Tq, H, D, Nc, Tkv, dtype, seed=51, unit=unit)
    nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    idx = gen.make_topk_idx(B, Tq, k, nv, seed=52, device=DEV)
    out, lse = lcsa.csa_sparse_attn(x["q"], x["ckv"], idx, x["kv"], x["sink"], q_pos0, 0, m, W, R, return_lse=True)
    ref, ref_lse = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), idx.cpu().numpy(), np64(x["kv"]), q_pos0, 0, m,
                                     W, _sink(x), R)
    assert_attn_close(np64(out).reshape(ref.shape), ref)
    np.testing.assert_allclose(np64(lse).reshape(ref_lse.shape), ref_lse, atol=2e-3)


@pytest.mark.parametrize("dtype,H,D,R,m,W,Tq,Nc,q_pos0,unit,sink", [
    ("fp32", 4, 64, 32, 128, 64, 300, 8, 724, True, True),
    ("bf16", 64, 512, 64, 128, 128, 130, 40, 2000, True, True),    # crosses a 128-block boundary
    ("bf16", 64, 512, 64, 128, 128, 130, 40, 2000, False, True),
    ("bf16", 64, 512, 64, 128, 128, 70, 40, 0, True, False),       # t < m: window only, no sink
    ("bf16", 64, 512, 64, 16, 128, 50, 400, 5000, True, True),     # many entries (> several tiles)
    ("bf16", 64, 512, 64, 128, 128, 160, 40, 4000, True, True),    # >= 296 rows: no key-range split
])
def test_hca_dense_attn_parity(lcsa, dtype, H, D, R, m, W, Tq, Nc, q_pos0, unit, sink):
    B = 2
    Tkv = q_pos0 + Tq
    x = _attn_case(B, Tq, H, D, Nc, Tkv, dtype, seed=61, unit=unit, sink=sink)
    out, lse = lcsa.hca_dense_attn(x["q"], x["ckv"], x["kv"], x["sink"], q_pos0, 0, m, W, R, return_lse=True)
    ref, ref_lse = O.hca_dense_attn(np64(x["q"]), np64(x["ckv"]), np64(x["kv"]), q_pos0, 0, m, W, _sink(x), R)
    assert_attn_close(np64(out).reshape(ref.shape), ref)
    np.testing.assert_allclose(np64(lse).reshape(ref_lse.shape), ref_lse, atol=2e-3)


def test_hca_causal_rows_from_position_zero(lcsa):
    """290 query rows at positions 0..289 with m = 1: every row a different
    number of visible entries, from none to 289."""
    B, H, D, R, m, W, Tq, Nc, q0 = 1, 64, 512, 64, 1, 128, 290, 290, 0
    x = _attn_case(B, Tq, H, D, Nc, q0 + Tq, "bf16", seed=63)
    out, lse = lcsa.hca_dense_attn(x["q"], x["ckv"], x["kv"], x["sink"], q0, 0, m, W, R, return_lse=True)
    ref, ref_lse = O.hca_dense_attn(np64(x["q"]), np64(x["ckv"]), np64(x["kv"]), q0, 0, m, W, _sink(x), R)
    assert_attn_close(np64(out).reshape(ref.shape), ref)
    np.testing.assert_allclose(np64(lse).reshape(ref_lse.shape), ref_lse, atol=2e-3)
    assert lcsa.get_device_status() == 0


def test_csa_key_range_splits_with_empty_items(lcsa):
    """40 early rows (positions 0..39, at most 9 visible entries) with k = 2048:
    the key range of k + window tiles is split three ways (few rows, long
    ranges), so most split items hold no keys and the persistent kernel's
    empty-item path writes them (zero partial output, -inf partial max) before
    the combine."""
    B, H, D, R, m, W, k, Tq, Nc, q0 = 1, 64, 512, 64, 4, 128, 2048, 40, 700, 0
    x = _attn_case(B, Tq, H, D, Nc, q0 + Tq, "bf16", seed=64)
    nv = [O.n_visible(q0 + i, m, Nc) for i in range(Tq)]
    idx = gen.make_topk_idx(B, Tq, k, nv, seed=65, device=DEV)
    out, lse = lcsa.csa_sparse_attn(x["q"], x["ckv"], idx, x["kv"], x["sink"], q0, 0, m, W, R, return_lse=True)
    ref, ref_lse = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), idx.cpu().numpy(), np64(x["kv"]), q0, 0, m, W,
                                     _sink(x), R)
    assert_attn_close(np64(out).reshape(ref.shape), ref)
    np.testing.assert_allclose(np64(lse).reshape(ref_lse.shape), ref_lse, atol=2e-3)
    assert lcsa.get_device_status() == 0


def test_decode_window_ring(lcsa):
    """Decode layout: kv holds only the last W raw rows (kv_pos0 = t-W+1)."""
    B, H, D, R, m, W, k, Nc = 3, 64, 512, 64, 4, 128, 512, 4000
    t = 4 * Nc
    x = _attn_case(B, 1, H, D, Nc, W, "bf16", seed=71)
    idx = gen.make_topk_idx(B, 1, k, [Nc], seed=72, device=DEV)
    out = lcsa.csa_sparse_attn(x["q"], x["ckv"], idx, x["kv"], x["sink"], t, t - W + 1, m, W, R)
    ref, _ = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), idx.cpu().numpy(), np64(x["kv"]), t, t - W + 1, m, W,
                               _sink(x), R)
    assert_attn_close(np64(out).reshape(ref.shape), ref)


def test_attn_bf16_output(lcsa):
    B, H, D, R, m, W, k, Tq, Nc, q0 = 1, 64, 512, 64, 4, 128, 128, 16, 600, 2400
    x = _attn_case(B, Tq, H, D, Nc, q0 + Tq, "bf16", seed=81)
    idx = gen.make_topk_idx(B, Tq, k, [O.n_visible(q0 + i, m, Nc) for i in range(Tq)], seed=82, device=DEV)
    out = lcsa.csa_sparse_attn(x["q"], x["ckv"], idx, x["kv"], x["sink"], q0, 0, m, W, R, out_dtype=torch.bfloat16)
    ref, _ = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), idx.cpu().numpy(), np64(x["kv"]), q0, 0, m, W,
                               _sink(x), R)
    assert_attn_close(np64(out).reshape(ref.shape), ref, max_abs=2e-2, mean_abs=3e-3)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_attn_output_alignment(lcsa, out_dtype):
    """An output buffer that is 16- but not 32-byte aligned takes the 16-byte
    store path and gives the same values as an aligned one."""
    B, H, D, R, m, W, Tq, Nc, q0 = 1, 64, 512, 64, 128, 128, 300, 40, 4800
    x = _attn_case(B, Tq, H, D, Nc, q0 + Tq, "bf16", seed=85)
    ref = lcsa.hca_dense_attn(x["q"], x["ckv"], x["kv"], x["sink"], q0, 0, m, W, R, out_dtype=out_dtype)
    shift = 16 // torch.tensor([], dtype=out_dtype).element_size()
    buf = torch.empty(B * Tq * H * D + 2 * shift, dtype=out_dtype, device=DEV)
    base = buf.data_ptr() % 32
    off = shift if base == 0 else 0                     # start 16 bytes past a 32-byte boundary
    out = buf[off:off + B * Tq * H * D].view(B, Tq, H, D)
    assert out.data_ptr() % 32 == 16
    lcsa.hca_dense_attn(x["q"], x["ckv"], x["kv"], x["sink"], q0, 0, m, W, R, out_dtype=out_dtype, out=out)
    assert torch.equal(out, ref)


def test_layer_shapes_use_tensor_cores(lcsa):
    x = _attn_case(1, 4, 64, 512, 100, 100, "bf16", seed=91)
    assert lcsa.attn_uses_tensor_cores(x["q"], x["ckv"], x["kv"], R=64)
    y = _attn_case(1, 4, 4, 64, 100, 100, "fp32", seed=92)
    assert not lcsa.attn_uses_tensor_cores(y["q"], y["ckv"], y["kv"], R=32)
    ix = gen.make_indexer_inputs(1, 4, 100, 64, 128, "bf16", seed=93, device=DEV)
    assert lcsa.indexer_uses_tensor_cores(ix["q_idx"], ix["k_idx"], 2048)


def test_device_status_clean(lcsa):
    torch.cuda.synchronize()
    assert lcsa.get_device_status() == 0


def test_bad_index_is_skipped_and_flagged(lcsa):
    """Every use of a selected index is checked before an address is formed:
    an index >= Nc is skipped (its slot is no key at all) and the device
    status reports LCSA_DEV_BAD_INDEX (2), read and cleared by the host; the
    next call on the same stream is clean.  Tensor-core shapes and the FP32
    CUDA-core kernel, with a row whose selection is entirely bad."""
    for dtype, H, D, R, k, Nc, q_pos0 in (("bf16", 64, 512, 64, 64, 500, 2400), ("fp32", 4, 64, 32, 16, 200, 900)):
        B, Tq, m, W = 1, 3, 4, 16
        x = _attn_case(B, Tq, H, D, Nc, q_pos0 + Tq, dtype, seed=96)
        nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
        idx = gen.make_topk_idx(B, Tq, k, nv, seed=97, device=DEV)
        assert lcsa.get_device_status() == 0
        bad = idx.clone()
        bad[0, 1, k - 1] = Nc + 7                      # last slot of row 1 points past the cache
        bad[0, 2, :] = Nc                              # every slot of row 2 (window and sink remain)
        out = lcsa.csa_sparse_attn(x["q"], x["ckv"], bad, x["kv"], x["sink"], q_pos0, 0, m, W, R)
        assert lcsa.get_device_status() == 2
        assert lcsa.get_device_status() == 0            # read and cleared
        sel = bad.cpu().numpy().copy()
        sel[sel >= Nc] = -1                             # the skipped slots are no keys
        ref, _ = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), sel, np64(x["kv"]), q_pos0, 0, m, W, _sink(x), R)
        assert_attn_close(np64(out).reshape(ref.shape), ref)
        out2 = lcsa.csa_sparse_attn(x["q"], x["ckv"], idx, x["kv"], x["sink"], q_pos0, 0, m, W, R)
        assert lcsa.get_device_status() == 0
        ref2, _ = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), idx.cpu().numpy(), np64(x["kv"]), q_pos0, 0, m, W,
                                    _sink(x), R)
        assert_attn_close(np64(out2).reshape(ref2.shape), ref2)
