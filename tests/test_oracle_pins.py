"""Pins for the CPU oracle: closed forms, brute force, a library attention
routine and values the pages print.  Each test targets a mistake that a
plausible bug in the oracle would make (dropped term, wrong sign or index,
transposed operand, off-by-one visibility)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- compress
@pytest.mark.parametrize("m,window", [(4, 8), (128, 128), (3, 6)])
def test_compress_equal_gates_is_block_mean(m, window):
    r = _rng(1)
    T, D = 10 * m + (m - 1), 7          # ragged tail: last partial block gets no entry
    kv = r.standard_normal((T, D))
    gate = np.tile(r.standard_normal((1, D)), (T, 1))  # equal over tokens, per channel
    out = O.compress(kv, gate, m, window)
    assert out.shape == (T // m, D)
    for j in range(T // m):
        lo, hi = max(0, (j + 1) * m - window), (j + 1) * m
        np.testing.assert_allclose(out[j], kv[lo:hi].mean(axis=0), rtol=0, atol=1e-13)


def test_csa_window_is_previous_plus_own_block():
    # one-hot gate: the single token with i % 2m == 1 dominates every 2m window
    m, T, D = 4, 64, 5
    r = _rng(2)
    kv = r.standard_normal((T, D))
    gate = np.where((np.arange(T) % (2 * m)) == 1, 80.0, 0.0)
    out = O.csa_compress(kv, gate, m)
    for j in range(T // m):
        lo, hi = max(0, (j - 1) * m), (j + 1) * m
        (star,) = [i for i in range(lo, hi) if i % (2 * m) == 1]
        np.testing.assert_allclose(out[j], kv[star], atol=1e-30 + 1e-12)


def test_hca_permutation_within_block_invariant():
    m, T, D = 16, 64, 6
    r = _rng(3)
    kv = r.standard_normal((T, D))
    gate = r.standard_normal((T, D))
    perm = np.concatenate([b * m + r.permutation(m) for b in range(T // m)])
    np.testing.assert_allclose(O.hca_compress(kv, gate, m), O.hca_compress(kv[perm], gate[perm], m),
                               atol=1e-13)


def test_compress_scalar_gate_is_broadcast():
    r = _rng(4)
    kv = r.standard_normal((40, 9))
    g = r.standard_normal(40)
    np.testing.assert_array_equal(O.csa_compress(kv, g, 4), O.csa_compress(kv, np.repeat(g[:, None], 9, 1), 4))


def test_compress_causal_prefix():
    r = _rng(5)
    kv = r.standard_normal((48, 4))
    gate = r.standard_normal((48, 4))
    base = O.csa_compress(kv, gate, 4)
    kv2, g2 = kv.copy(), gate.copy()
    kv2[24:] += 5.0
    g2[24:] -= 3.0
    out2 = O.csa_compress(kv2, g2, 4)
    np.testing.assert_array_equal(base[:6], out2[:6])     # entry 5 pools tokens 16..23
    assert not np.allclose(base[6], out2[6])              # entry 6 pools 20..27


def test_compress_rmsnorm_unit_rms():
    r = _rng(6)
    kv = r.standard_normal((32, 16))
    gate = r.standard_normal((32, 16))
    out = O.csa_compress(kv, gate, 4, rms_weight=np.full(16, 2.0), rms_eps=0.0)
    np.testing.assert_allclose(np.sqrt((out ** 2).mean(axis=1)), 2.0, rtol=1e-12)


def test_entry_counts_golden():
    """1M tokens give 250K CSA entries and about 7,800 HCA entries."""
    g = json.load(open(os.path.join(GOLD, "entry_counts.json")))
    T = g["T"]
    z = np.zeros((T, 1))
    assert O.csa_compress(z, z[:, 0], g["csa_m"]).shape[0] == g["csa_entries"]
    hca = O.hca_compress(z, z[:, 0], g["hca_m"]).shape[0]
    assert abs(hca - g["hca_entries_approx"]) / g["hca_entries_approx"] < g["approx_rel_tol"]


# ---------------------------------------------------------------- indexer
def test_indexer_single_head_bruteforce():
    r = _rng(7)
    Tq, Nc, D_I, m, q_pos0 = 6, 9, 5, 4, 20
    q = r.standard_normal((Tq, 1, D_I))
    k = r.standard_normal((Nc, D_I))
    w = np.ones((Tq, 1))
    s = O.indexer_scores(q, w, k, q_pos0, m)
    for i in range(Tq):
        t = q_pos0 + i
        for j in range(Nc):
            if j < t // m:
                dot = math.fsum(float(q[i, 0, d]) * float(k[j, d]) for d in range(D_I))
                assert s[i, j] == pytest.approx(max(0.0, dot), abs=1e-12)
            else:
                assert s[i, j] == -np.inf


def test_indexer_relu_per_head_then_weighted_sum():
    r = _rng(8)
    Tq, H, Nc, D_I = 3, 4, 12, 6
    q = r.standard_normal((Tq, H, D_I))
    k = r.standard_normal((Nc, D_I))
    w1 = r.standard_normal((Tq, H))
    w2 = r.standard_normal((Tq, H))
    s1 = O.indexer_scores(q, w1, k, 100, 4)
    s2 = O.indexer_scores(q, w2, k, 100, 4)
    s12 = O.indexer_scores(q, w1 + w2, k, 100, 4)
    np.testing.assert_allclose(s12, s1 + s2, atol=1e-12)       # linear in w => ReLU is per head
    # a single head with weight -1 gives -relu(dot): never positive
    s_neg = O.indexer_scores(q[:, :1], -np.ones((Tq, 1)), k, 100, 4)
    assert (s_neg <= 0).all()
    # heads are a set: permuting heads of q and w together changes nothing
    p = r.permutation(H)
    np.testing.assert_allclose(O.indexer_scores(q[:, p], w1[:, p], k, 100, 4), s1, atol=1e-12)


# ---------------------------------------------------------------- FP4 (MXFP4) indexer path
def _e2m1_from_bits(c):
    """Value of a 4-bit E2M1 code decoded from its fields: sign bit 3,
    exponent bits 2-1 (bias 1), mantissa bit 0; exponent 0 is subnormal."""
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_codes_bruteforce_from_bit_fields():
    # every multiple of 1/32 in [-8, 8]: nearest code of the same sign, ties to
    # an even mantissa bit (round to nearest even), large magnitudes saturate
    for n in range(-256, 257):
        y = n / 32.0
        cands = [c for c in range(16) if ((c >> 3) & 1) == (1 if y < 0 else 0)]
        best = min(abs(y - _e2m1_from_bits(c)) for c in cands)
        near = [c for c in cands if abs(y - _e2m1_from_bits(c)) == best]
        want = near[0] if len(near) == 1 else [c for c in near if c % 2 == 0][0]
        assert O.e2m1_code(y) == want, y


def test_mx_round_to_nearest_even_midpoints():
    # midpoints of the E2M1 grid go to the neighbour with the even mantissa
    # bit; 7 saturates to 6 (the block's amax 7 fixes X = 0)
    y = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.75, -5.0]
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, -1.0, -4.0]
    x = np.zeros((1, 32))
    x[0, :len(y)] = y
    c, sc = O.quantize_mxfp4(x)
    assert sc[0, 0] == 127
    np.testing.assert_array_equal(O.dequantize_mxfp4(c, sc)[0, :len(y)], want)


def test_mx_scale_rule():
    # X = floor(log2(amax)) - 2, clamped to [-127, 127]; UE8M0 byte = X + 127
    for amax, byte in [(1.0, 125), (6.0, 127), (7.999, 127), (8.0, 128), (0.75, 124),
                       (2.0 ** -130, 0), (0.0, 0), (2.0 ** 126, 251)]:
        x = np.zeros((1, 32))
        x[0, 5] = amax
        assert O.quantize_mxfp4(x)[1][0, 0] == byte, amax
    x = np.zeros((1, 64))
    x[0, 40] = np.inf
    c, sc = O.quantize_mxfp4(x)
    assert sc[0, 1] == 255 and not c[0, 16:].any() and sc[0, 0] == 0


def test_mx_roundtrip_of_representable_blocks():
    r = _rng(21)
    codes = r.integers(0, 256, (6, 64), dtype=np.uint8)
    codes[:, ::16] = (codes[:, ::16] & 0xF0) | 0x7        # element 0 of every block = +6: X recovers
    scales = r.integers(100, 140, (6, 4), dtype=np.uint8)
    v = O.dequantize_mxfp4(codes, scales)
    c2, s2 = O.quantize_mxfp4(v)
    np.testing.assert_array_equal(s2, scales)
    # codes agree up to the sign of zero (a -0 input quantises to +0)
    np.testing.assert_array_equal(O.dequantize_mxfp4(c2, s2), v)


def test_mx_error_within_half_spacing():
    r = _rng(22)
    x = r.standard_normal((40, 128)) * np.exp2(r.integers(-20, 20, (40, 1)))
    c, sc = O.quantize_mxfp4(x)
    d = O.dequantize_mxfp4(c, sc)
    X = np.repeat(sc.astype(np.float64) - 127, 32, axis=1)
    y = np.abs(x) / np.exp2(X)
    half = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    err = np.abs(x - d) / np.exp2(X)
    inside = y <= 6
    assert (err[inside] <= half[inside] + 1e-12).all()
    # amax / 2^X lies in [4, 8): magnitudes above 6 saturate to 6
    assert (y < 8).all() and (np.abs(d[~inside]) / np.exp2(X[~inside]) == 6.0).all()
    assert (np.sign(d) * np.sign(x) >= 0).all()


def test_indexer_mxfp4_exact_on_representable_inputs():
    # quantisation is the identity on values already on the MXFP4 grid with a
    # full-range element per block, so the FP4 path reduces to the exact indexer
    r = _rng(23)
    Tq, H, Nc, D_I, m, q_pos0 = 3, 4, 40, 64, 4, 150

    def grid(shape):
        c = r.integers(0, 256, shape[:-1] + (shape[-1] // 2,), dtype=np.uint8)
        c[..., ::16] = (c[..., ::16] & 0xF0) | 0x6         # a +4 in every block
        sc = r.integers(118, 128, shape[:-1] + (shape[-1] // 32,), dtype=np.uint8)
        return c, sc

    qc, qs = grid((Tq, H, D_I))
    kc, ks = grid((Nc, D_I))
    q = O.dequantize_mxfp4(qc, qs)
    k = O.dequantize_mxfp4(kc, ks)
    w = r.standard_normal((Tq, H))
    s_fp4 = O.indexer_scores_mxfp4(q, w, kc, ks, q_pos0, m)
    s_ref = O.indexer_scores(q, w, k, q_pos0, m)
    np.testing.assert_array_equal(s_fp4, s_ref)
    idx, _ = O.indexer_topk_mxfp4(q, w, kc, ks, q_pos0, m, 8)
    idx_ref, _ = O.indexer_topk(q, w, k, q_pos0, m, 8)
    np.testing.assert_array_equal(idx, idx_ref)


def test_indexer_mxfp4_quantises_the_query():
    # a query off the grid scores as its rounded copy does
    r = _rng(24)
    q = r.standard_normal((2, 3, 32))
    k_raw = r.standard_normal((10, 32))
    kc, ks = O.quantize_mxfp4(k_raw)
    w = r.standard_normal((2, 3))
    qc, qs = O.quantize_mxfp4(q)
    a = O.indexer_scores_mxfp4(q, w, kc, ks, 44, 4)
    b = O.indexer_scores(O.dequantize_mxfp4(qc, qs), w, O.dequantize_mxfp4(kc, ks), 44, 4)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, O.indexer_scores(q, w, O.dequantize_mxfp4(kc, ks), 44, 4))


def test_visibility_boundary():
    # j visible iff j < floor(t/m): m=4 -> t=0..3 see 0, t=4..7 see 1, t=8 sees 2
    assert [O.n_visible(t, 4, 100) for t in range(10)] == [0, 0, 0, 0, 1, 1, 1, 1, 2, 2]
    assert O.n_visible(10 ** 6, 4, 250000) == 250000
    assert O.n_visible(127, 128, 8) == 0 and O.n_visible(128, 128, 8) == 1


# ---------------------------------------------------------------- top-k
def test_topk_golden_toy():
    g = json.load(open(os.path.join(GOLD, "topk_toy.json")))
    assert list(O.topk_select(g["scores"], g["k"])) == g["expected_idx"]


def test_topk_all_equal_and_short_rows():
    assert list(O.topk_select(np.full(10, 0.5), 4)) == [0, 1, 2, 3]
    assert list(O.topk_select(np.array([3.0, 1.0, 2.0]), 5)) == [0, 1, 2, -1, -1]
    # signed zeros are equal: ties go to the lower index
    assert list(O.topk_select(np.array([-0.0, 0.0, -1.0, -0.0]), 2)) == [0, 1]


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce_subsets(seed):
    r = _rng(100 + seed)
    n, k = 9, 4
    row = np.round(r.standard_normal(n) * 2) / 2        # frequent ties
    def beats(i, j):                                     # i ranks above j
        return row[i] > row[j] or (row[i] == row[j] and i < j)
    valid = [S for S in itertools.combinations(range(n), k)
             if all(beats(i, j) for i in S for j in range(n) if j not in S)]
    assert len(valid) == 1
    assert list(O.topk_select(row, k)) == list(valid[0])


def test_topk_from_scores_respects_n_valid():
    s = np.array([[5.0, 4.0, 3.0, 9.0], [1.0, 2.0, 3.0, 4.0]])
    out = O.topk_from_scores(s, [2, 0], 3)
    assert out.tolist() == [[0, 1, -1], [-1, -1, -1]]


# ---------------------------------------------------------------- rope
def test_rope_matches_complex_rotation():
    r = _rng(9)
    D, R = 12, 8
    x = r.standard_normal((3, D))
    pos = np.array([0.0, 5.0, 1234567.0])
    y = O.rope_rotate(x, pos, R, 10000.0)
    np.testing.assert_array_equal(y[:, :D - R], x[:, :D - R])
    z = x[:, D - R::2] + 1j * x[:, D - R + 1::2]
    theta = 10000.0 ** (-np.arange(R // 2) * 2.0 / R)
    zr = z * np.exp(1j * pos[:, None] * theta[None, :])
    np.testing.assert_allclose(y[:, D - R::2], zr.real, atol=1e-9)
    np.testing.assert_allclose(y[:, D - R + 1::2], zr.imag, atol=1e-9)
    np.testing.assert_allclose(O.rope_rotate(y, -pos, R), x, atol=1e-9)


# ---------------------------------------------------------------- attention
def _complex_rot(x, pos, R, base=10000.0):
    """Independent restatement of the rotary map through complex numbers."""
    x = np.array(x, dtype=np.float64)
    D = x.shape[-1]
    if R == 0:
        return x
    z = x[..., D - R::2] + 1j * x[..., D - R + 1::2]
    theta = base ** (-np.arange(R // 2) * 2.0 / R)
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * theta)
    y = x.copy()
    y[..., D - R::2] = z.real
    y[..., D - R + 1::2] = z.imag
    return y


@pytest.mark.parametrize("R", [0, 8])
def test_m1_window1_reduces_to_causal_sdpa(R):
    """m=1, W=1, no sink: HCA is ordinary causal single-KV-head attention."""
    r = _rng(10 + R)
    T, H, D = 17, 3, 16
    kv = r.standard_normal((1, T, D))
    q = r.standard_normal((1, T, H, D))
    ckv = O.hca_compress(kv[0], r.standard_normal((T, D)), 1)[None]   # m=1: entries are the tokens
    np.testing.assert_array_equal(ckv[0], kv[0])
    out, lse = O.hca_dense_attn(q, ckv, kv, 0, 0, 1, 1, None, R)
    pos = np.arange(T)
    qr = torch.from_numpy(_complex_rot(q[0], pos[:, None], R)).permute(1, 0, 2)   # [H,T,D]
    kr = torch.from_numpy(_complex_rot(kv[0], pos, R))[None].expand(H, T, D)
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, kr, is_causal=True)
    ref = _complex_rot(ref.permute(1, 0, 2).numpy(), -pos[:, None], R)
    np.testing.assert_allclose(out, ref, atol=1e-12)
    logits = torch.einsum("htd,sd->hts", qr, kr[0]) / math.sqrt(D)
    mask = torch.triu(torch.ones(T, T, dtype=torch.bool), 1)
    ref_lse = torch.logsumexp(logits.masked_fill(mask, -float("inf")), dim=-1).T.numpy()
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12)


def test_sink_closed_form_zero_query():
    r = _rng(11)
    H, D, T = 2, 8, 40
    kv = r.standard_normal((1, T, D))
    ckv = r.standard_normal((1, T // 4, D))
    sink = np.array([0.7, -1.3])
    q = np.zeros((1, 1, H, D))
    t = 25
    n_keys = O.n_visible(t, 4, T // 4) + 8            # entries 0..5 plus window of 8 raw tokens
    out, lse = O.hca_dense_attn(q, ckv, kv, t, 0, 4, 8, sink, R=0, rows=[(0, 0)])
    expect = (ckv[0, :6].sum(0) + kv[0, t - 7:t + 1].sum(0))[None, :] / (n_keys + np.exp(sink))[:, None]
    np.testing.assert_allclose(out[0], expect, atol=1e-13)
    np.testing.assert_allclose(lse[0], np.log(n_keys + np.exp(sink)), atol=1e-13)


def test_sink_weights_sum_below_one():
    r = _rng(12)
    H, D = 3, 8
    u = r.standard_normal(D)
    kv = np.tile(u, (1, 20, 1))
    ckv = np.tile(u, (1, 5, 1))
    q = r.standard_normal((1, 1, H, D))
    for sink, lo, hi in [(np.zeros(H), 0.0, 1.0), (np.full(H, -1e3), 1 - 1e-12, 1 + 1e-12)]:
        out, _ = O.hca_dense_attn(q, ckv, kv, 19, 0, 4, 4, sink, R=0, rows=[(0, 0)])
        ratio = out[0] / u[None, :]
        assert (ratio > lo).all() and (ratio < hi).all()
    out, _ = O.hca_dense_attn(q, ckv, kv, 19, 0, 4, 4, None, R=0, rows=[(0, 0)])
    np.testing.assert_allclose(out[0] / u[None, :], 1.0, atol=1e-12)


def test_single_window_key_closed_form():
    """No visible entry and W=1: out = kv_t * sigmoid(l - sigma) with the
    relative-position logit l = q.kv_t/sqrt(D) (the -t rotation cancels)."""
    r = _rng(13)
    H, D, R = 2, 16, 8
    kv = r.standard_normal((1, 3, D))
    q = r.standard_normal((1, 1, H, D))
    sink = np.array([0.3, -0.4])
    t = 2                                      # t < m: no entry visible
    out, _ = O.hca_dense_attn(q, np.zeros((1, 0, D)), kv, t, 0, 4, 1, sink, R, rows=[(0, 0)])
    lg = q[0, 0] @ kv[0, t] / math.sqrt(D)
    expect = kv[0, t][None, :] / (1.0 + np.exp(sink - lg))[:, None]
    np.testing.assert_allclose(out[0], expect, atol=1e-12)


def test_csa_translation_invariance():
    """Shift every position by delta (a multiple of m): entries move by delta/m,
    the window rows and the query by delta; the output does not change."""
    r = _rng(14)
    H, D, R, m, W = 2, 16, 8, 4, 6
    Nc, Tkv, k = 30, 130, 8
    ckv = r.standard_normal((1, Nc, D))
    kv = r.standard_normal((1, Tkv, D))
    q = r.standard_normal((1, 3, H, D))
    sink = r.standard_normal(H)
    idx = np.stack([np.sort(r.choice(n, k, replace=False)) for n in (25, 26, 27)])[None]
    out0, lse0 = O.csa_sparse_attn(q, ckv, idx, kv, 101, 0, m, W, sink, R)
    dshift = 12
    ckv2 = np.concatenate([r.standard_normal((1, dshift // m, D)), ckv], axis=1)
    out1, lse1 = O.csa_sparse_attn(q, ckv2, idx + dshift // m, kv, 101 + dshift, dshift, m, W, sink, R)
    np.testing.assert_allclose(out1, out0, atol=1e-9)
    np.testing.assert_allclose(lse1, lse0, atol=1e-9)


def test_csa_with_all_visible_selected_equals_dense():
    r = _rng(15)
    H, D, R, m, W = 2, 16, 8, 4, 5
    T = 64
    ckv = r.standard_normal((1, T // m, D))
    kv = r.standard_normal((1, T, D))
    q = r.standard_normal((1, T, H, D))
    sink = r.standard_normal(H)
    k = T // m
    idx = np.full((1, T, k), -1)
    for t in range(T):
        nv = O.n_visible(t, m, T // m)
        idx[0, t, :nv] = np.arange(nv)
    a, la = O.csa_sparse_attn(q, ckv, idx, kv, 0, 0, m, W, sink, R)
    b, lb = O.hca_dense_attn(q, ckv, kv, 0, 0, m, W, sink, R)
    np.testing.assert_allclose(a, b, atol=1e-13)
    np.testing.assert_allclose(la, lb, atol=1e-13)


def test_decode_ring_equals_full_kv():
    r = _rng(16)
    H, D, R, W, T = 2, 16, 8, 8, 50
    kv = r.standard_normal((1, T, D))
    ckv = r.standard_normal((1, T // 4, D))
    q = r.standard_normal((1, 1, H, D))
    t = T - 1
    full, _ = O.hca_dense_attn(q, ckv, kv, t, 0, 4, W, None, R)
    ring, _ = O.hca_dense_attn(q, ckv, kv[:, t - W + 1:], t, t - W + 1, 4, W, None, R)
    np.testing.assert_array_equal(full, ring)


def test_hca_pipeline_strictly_causal():
    r = _rng(17)
    H, D, R, m, W, T = 2, 8, 4, 8, 4, 64
    kv = r.standard_normal((1, T, D))
    gate = r.standard_normal((1, T, D))
    q = r.standard_normal((1, T, H, D))
    def run(kv_, gate_):
        ckv = O.hca_compress(kv_[0], gate_[0], m)[None]
        return O.hca_dense_attn(q, ckv, kv_, 0, 0, m, W, None, R)[0]
    base = run(kv, gate)
    kv2, g2 = kv.copy(), gate.copy()
    kv2[0, 30:] += 1.0
    g2[0, 30:] += 2.0
    out2 = run(kv2, g2)
    np.testing.assert_array_equal(base[:30], out2[:30])
    assert not np.allclose(base[30], out2[30])


# ---------------------------------------------------------------- grouped output projection
def test_round_bf16_matches_fp32_rounding_and_ties():
    # inputs that are FP32 values round in one step, so torch's FP32 -> BF16 is the reference
    r = _rng(31)
    x = (r.standard_normal(20000) * np.exp2(r.integers(-120, 120, 20000))).astype(np.float32).astype(np.float64)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O._round_bf16(x), ref)
    # exact midpoints go to the even neighbour; BF16 values stay put
    np.testing.assert_array_equal(O._round_bf16(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(2 + 2.0 ** -7), 1.5])),
                                  [1.0, 1 + 2.0 ** -6, -2.0, 1.5])


def test_grouped_out_proj_equals_composed_dense_projection():
    # without the BF16 intermediate the grouped projection is one linear map:
    # W_out . blockdiag(W_group[0..g-1]) applied to the flattened head outputs
    r = _rng(32)
    T, n_h, c, g, d_g, d = 5, 8, 16, 4, 12, 20
    o = r.standard_normal((T, n_h, c))
    w1 = r.standard_normal((g, d_g, n_h // g * c))
    w2 = r.standard_normal((d, g * d_g))
    kg = n_h // g * c
    bd = np.zeros((g * d_g, n_h * c))
    for j in range(g):
        bd[j * d_g:(j + 1) * d_g, j * kg:(j + 1) * kg] = w1[j]
    np.testing.assert_allclose(O.grouped_out_proj(o, w1, w2, round_mid=False), o.reshape(T, -1) @ (w2 @ bd).T,
                               rtol=1e-12, atol=1e-12)


def test_grouped_out_proj_single_identity_group_is_plain_projection():
    r = _rng(33)
    T, n_h, c, d = 4, 2, 8, 6
    o = torch.randn(T, n_h, c, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).double().numpy()
    w2 = r.standard_normal((d, n_h * c))
    y = O.grouped_out_proj(o, np.eye(n_h * c)[None], w2)       # BF16 inputs: the BF16 intermediate is exact
    np.testing.assert_allclose(y, o.reshape(T, -1) @ w2.T, rtol=1e-13, atol=1e-13)


def test_grouped_out_proj_group_permutation():
    r = _rng(34)
    T, n_h, c, g, d_g, d = 3, 8, 4, 4, 5, 7
    o = r.standard_normal((T, n_h, c))
    w1 = r.standard_normal((g, d_g, n_h // g * c))
    w2 = r.standard_normal((d, g * d_g))
    p = np.array([2, 0, 3, 1])
    hp = np.concatenate([np.arange(j * (n_h // g), (j + 1) * (n_h // g)) for j in p])
    cp = np.concatenate([np.arange(j * d_g, (j + 1) * d_g) for j in p])
    np.testing.assert_allclose(O.grouped_out_proj(o[:, hp], w1[p], w2[:, cp], round_mid=False),
                               O.grouped_out_proj(o, w1, w2, round_mid=False), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- FP8 entry cache
def test_e4m3_codes_bruteforce_over_all_codes():
    # nearest of the 254 finite codes of the same sign, ties to an even mantissa,
    # saturation at 448; values on a fine grid around every binade
    cands = [c for c in range(256) if (c & 0x7F) != 0x7F]
    vals = {c: O.e4m3_value(c) for c in cands}
    ys = [s * m * 2.0 ** k for s in (1, -1) for k in range(-12, 10) for m in np.arange(1, 2, 1 / 64)]
    ys += [0.0, 448.0, 460.0, 1e6, -1e6]
    got = O.e4m3_codes(np.array(ys))
    for y, c in zip(ys, got):
        same = [cc for cc in cands if (cc >> 7) == (1 if y < 0 else 0)]
        a = min(abs(y), 448.0)
        best = min(abs(a - abs(vals[cc])) for cc in same)
        near = [cc for cc in same if abs(a - abs(vals[cc])) == best]
        want = near[0] if len(near) == 1 else [cc for cc in near if cc % 2 == 0][0]
        assert int(c) == want, y


def test_e4m3_values_closed_forms():
    assert O.e4m3_value(0x7E) == 448.0 and O.e4m3_value(0x01) == 2.0 ** -9 and O.e4m3_value(0x38) == 1.0
    assert O.e4m3_value(0xB8) == -1.0 and np.isnan(O.e4m3_value(0x7F)) and np.isnan(O.e4m3_value(0xFF))
    assert (np.diff(O.E4M3_POS) > 0).all()


def test_fp8_entry_scale_rule_and_rope_passthrough():
    r = _rng(41)
    D, R = 512, 64
    x = r.standard_normal((6, D)) * np.exp2(r.integers(-12, 12, (6, 1)))
    x[1, :D - R] = 0.0                          # all-zero body
    x[2, 7] = 448.0 * 2.0 ** -3                 # amax exactly 448 * 2^-3 -> X = -3
    x[2, :D - R] = np.clip(x[2, :D - R], -56.0, 56.0)
    codes, sc, rope = O.quantize_entries_fp8(x, R)
    X = sc.astype(np.int64) - 127
    amax = np.abs(x[:, :D - R]).max(axis=1)
    for i in range(6):
        if amax[i] == 0:
            assert X[i] == -124 and not codes[i].any()
        else:
            assert amax[i] <= 448.0 * 2.0 ** X[i] and amax[i] > 448.0 * 2.0 ** (X[i] - 1)
    assert X[2] == -3
    np.testing.assert_array_equal(rope, O._round_bf16(x[:, D - R:]))
    d = O.dequantize_entries_fp8(codes, sc, rope)
    np.testing.assert_array_equal(d[:, D - R:], rope)
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 on normals, absolute <= 2^-10 * 2^X below
    err = np.abs(d[:, :D - R] - x[:, :D - R])
    bound = np.maximum(np.abs(x[:, :D - R]) * 2.0 ** -4, 2.0 ** -10 * np.exp2(X)[:, None])
    assert (err <= bound + 1e-300).all()


def test_fp8_entry_roundtrip_of_representable_entries():
    # entries already on the scaled E4M3 grid with the saturating code present come back unchanged
    r = _rng(42)
    codes = r.integers(0, 0x7F, (4, 448)).astype(np.uint8)
    codes = np.where((codes & 0x7F) == 0x7F, 0x7E, codes).astype(np.uint8)
    codes[:, 0] = 0x7E                          # every entry holds +448 * 2^X
    codes |= (r.integers(0, 2, (4, 448)) << 7).astype(np.uint8)
    codes[:, 0] &= 0x7F
    sc = r.integers(100, 130, 4).astype(np.uint8)
    rope = O._round_bf16(r.standard_normal((4, 64)))
    x = O.dequantize_entries_fp8(codes, sc, rope)
    c2, s2, r2 = O.quantize_entries_fp8(x, 64)
    np.testing.assert_array_equal(s2, sc)
    np.testing.assert_array_equal(O.dequantize_entries_fp8(c2, s2, r2), x)


def test_fp8_entry_tiny_magnitudes_stay_exact_in_bf16():
    # entries far below 448 * 2^-124 take the floor scale X = -124: their codes
    # are E4M3 subnormals or zero, and every dequantised value is a BF16 number
    # (multiples of 2^-133), checked against an independent BF16 rounding
    r = _rng(43)
    D, R = 512, 64
    x = r.standard_normal((3, D))
    x[0, :D - R] *= 2.0 ** -128                   # amax ~ 2^-126: normal FP64, far below the floor
    x[1, :D - R] *= 2.0 ** -130
    x[2, :D - R] = 0.0
    x[2, 5] = 2.0 ** -133                         # one BF16-subnormal-sized value
    codes, sc, rope = O.quantize_entries_fp8(x, R)
    assert (sc.astype(np.int64) - 127 == -124).all()
    d = O.dequantize_entries_fp8(codes, sc, rope)
    body = d[:, :D - R]
    np.testing.assert_array_equal(body, O._round_bf16(body))
    assert (np.abs(np.rint(body * 2.0 ** 133) - body * 2.0 ** 133) == 0).all()
    # the one value of row 2 is the E4M3 code 2^-9 times 2^-124
    assert codes[2, 5] == 0x01 and d[2, 5] == 2.0 ** -133
    # E4M3 error bound at the floor scale: 2^-4 relative on normals, half the
    # subnormal spacing (2^-10 * 2^-124) below
    err = np.abs(body - x[:, :D - R])
    assert (err <= np.maximum(np.abs(x[:, :D - R]) * 2.0 ** -4, 2.0 ** -134)).all()
