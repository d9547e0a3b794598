"""The FP8 entry cache (E4M3 body with one power-of-two scale per entry, BF16
rotary dims): the library's quantiser against the oracle bit for bit, and the
core attention over the cache against the oracle's attention over the
dequantised entries (and, bit for bit, against the BF16 attention over the
same entries expanded to BF16, which is exact)."""
import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as O
from workloads import gen

pytestmark = pytest.mark.gpu

DEV = "cuda"
ATT_MAX, ATT_MEAN = 1e-2, 1e-3


@pytest.fixture(scope="module")
def lcsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_library
    return build_library()


def np64(t):
    return t.detach().double().cpu().numpy()


def _entries(dtype, seed):
    """Entry rows [40, 512] with the edge cases of the scale and code rules."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(40, 512, generator=g) * torch.exp2(torch.randint(-20, 20, (40, 1), generator=g).float())
    x[0, :448] = 0.0                                    # all-zero body: floor scale
    x[1, :448] = -0.0                                   # negative zeros code +0
    x[2, :448] = torch.randn(448, generator=g) * 2.0 ** -130   # below the floor: E4M3 subnormals / zeros
    x[3, :448] = 0.0
    x[3, 9] = 448.0 * 2.0 ** -3                        # amax exactly 448 * 2^X
    # E4M3 midpoints after scaling by 2^X (X = 0 with amax 448): ties to an even code
    mids = torch.tensor([1.0625, 1.1875, 0.5 * (2 ** -9), 1.5 * 2 ** -9, 3.0 * 2 ** -10, 448.0, 240.0, 232.0,
                         -1.0625, -0.5 * (2 ** -9)])
    x[4, :448] = 1.0
    x[4, 0] = 448.0
    x[4, 1:1 + len(mids)] = mids
    x[5, :448] = x[5, :448] * 1e-3
    x[5, 3] = -2.0 ** -140                             # tiny negative next to O(1e-3) values
    return x.to(torch.float32 if dtype == "fp32" else torch.bfloat16)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_quantize_entries_fp8_bit_exact(lcsa, dtype):
    x = _entries(dtype, 81)
    codes, scales, rope = lcsa.quantize_entries_fp8(x.to(DEV), 64)
    rc, rs, rr = O.quantize_entries_fp8(x.double().numpy(), 64)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(np64(rope), rr)
    # the expansion the attention kernel performs is exact: a BF16 tensor
    d = O.dequantize_entries_fp8(rc, rs, rr)
    np.testing.assert_array_equal(torch.tensor(d).to(torch.bfloat16).double().numpy(), d)


def _dequant_bf16(cache):
    codes, scales, rope = (t.cpu().numpy() if t.dtype == torch.uint8 else np64(t) for t in cache)
    d = O.dequantize_entries_fp8(codes, scales, rope)
    return d, torch.tensor(d, dtype=torch.float64).to(torch.bfloat16).to(DEV)


def _assert_close(got, ref):
    err = np.abs(np64(got).reshape(ref.shape) - ref)
    assert err.max() <= ATT_MAX, f"max abs err {err.max():.3e}"
    assert err.mean() <= ATT_MEAN, f"mean abs err {err.mean():.3e}"


@pytest.mark.parametrize("k,Tq,Nc,q_pos0,unit", [
    (256, 40, 700, 2700, True),       # layer shapes, several tiles
    (256, 40, 700, 2700, False),      # spec scale
    (2048, 9, 3000, 9000, True),      # full k
    (100, 20, 900, 3000, True),       # odd k: ragged last tile
    (3000, 4, 5000, 19000, True),     # k > 2048: forced key-range splits
    (2048, 3, 20000, 80000, True),    # few rows (slot-indexed rotary slices)
])
def test_csa_sparse_attn_fp8_parity(lcsa, k, Tq, Nc, q_pos0, unit):
    B, H, D, R, m, W = 2, 64, 512, 64, 4, 128
    Tkv = q_pos0 + Tq
    x = gen.make_attn_inputs(B, Tq, H, D, Nc, Tkv, "bf16", seed=91, device=DEV, unit_scale=unit)
    nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    idx = gen.make_topk_idx(B, Tq, k, nv, seed=92, device=DEV)
    cache = lcsa.quantize_entries_fp8(x["ckv"], R)
    d, d_bf16 = _dequant_bf16(cache)
    out, lse = lcsa.csa_sparse_attn_fp8(x["q"], cache, idx, x["kv"], x["sink"], q_pos0, 0, m, W, R,
                                        return_lse=True)
    ref, ref_lse = O.csa_sparse_attn(np64(x["q"]), d, idx.cpu().numpy(), np64(x["kv"]), q_pos0, 0, m, W,
                                     np64(x["sink"]), R)
    _assert_close(out, ref)
    np.testing.assert_allclose(np64(lse).reshape(ref_lse.shape), ref_lse, atol=2e-3)
    # the same kernel on the expanded BF16 entries gives the same bits
    out16 = lcsa.csa_sparse_attn(x["q"], d_bf16, idx, x["kv"], x["sink"], q_pos0, 0, m, W, R)
    assert torch.equal(out, out16)
    assert lcsa.get_device_status() == 0


@pytest.mark.parametrize("m,Tq,Nc,q_pos0,unit", [
    (128, 130, 40, 2000, True),       # crosses a 128-block boundary
    (128, 130, 40, 2000, False),
    (16, 50, 400, 5000, True),        # many entries
    (128, 160, 40, 4000, True),       # >= 296 rows: no key-range split
    (128, 70, 40, 0, True),           # t < m: window only
])
def test_hca_dense_attn_fp8_parity(lcsa, m, Tq, Nc, q_pos0, unit):
    B, H, D, R, W = 2, 64, 512, 64, 128
    Tkv = q_pos0 + Tq
    x = gen.make_attn_inputs(B, Tq, H, D, Nc, Tkv, "bf16", seed=93, device=DEV, unit_scale=unit)
    cache = lcsa.quantize_entries_fp8(x["ckv"], R)
    d, d_bf16 = _dequant_bf16(cache)
    out, lse = lcsa.hca_dense_attn_fp8(x["q"], cache, x["kv"], x["sink"], q_pos0, 0, m, W, R, return_lse=True)
    ref, ref_lse = O.hca_dense_attn(np64(x["q"]), d, np64(x["kv"]), q_pos0, 0, m, W, np64(x["sink"]), R)
    _assert_close(out, ref)
    np.testing.assert_allclose(np64(lse).reshape(ref_lse.shape), ref_lse, atol=2e-3)
    out16 = lcsa.hca_dense_attn(x["q"], d_bf16, x["kv"], x["sink"], q_pos0, 0, m, W, R)
    assert torch.equal(out, out16)
    assert lcsa.get_device_status() == 0


def test_fp8_cache_bad_index_is_skipped_and_flagged(lcsa):
    """An index >= Nc in the selection is skipped (its slot contributes
    nothing) and the device status reports LCSA_DEV_BAD_INDEX (2)."""
    B, Tq, H, D, R, m, W, k, Nc, q_pos0 = 1, 3, 64, 512, 64, 4, 128, 64, 500, 2400
    x = gen.make_attn_inputs(B, Tq, H, D, Nc, q_pos0 + Tq, "bf16", seed=94, device=DEV, unit_scale=True)
    nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    idx = gen.make_topk_idx(B, Tq, k, nv, seed=95, device=DEV)
    assert lcsa.get_device_status() == 0
    bad = idx.clone()
    bad[0, 1, k - 1] = Nc + 7                            # last slot of row 1 points past the cache
    bad[0, 2, :] = Nc                                    # every slot of row 2
    cache = lcsa.quantize_entries_fp8(x["ckv"], R)
    out = lcsa.csa_sparse_attn_fp8(x["q"], cache, bad, x["kv"], x["sink"], q_pos0, 0, m, W, R)
    assert lcsa.get_device_status() == 2
    assert lcsa.get_device_status() == 0                 # read and cleared
    d, _ = _dequant_bf16(cache)
    sel = bad.cpu().numpy().copy()
    sel[sel >= Nc] = -1                                  # the skipped slots are no keys at all
    ref, _ = O.csa_sparse_attn(np64(x["q"]), d, sel, np64(x["kv"]), q_pos0, 0, m, W, np64(x["sink"]), R)
    _assert_close(out, ref)
