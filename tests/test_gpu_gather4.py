"""CSA sparse attention with its selected rows staged by TMA tile::gather4
(lcsa_set_attn_gather(1)) instead of 16-byte cp.async: parity with the oracle
on the layer shapes, the decode layout (rotary slices per query slot), key-
range splits and bad indices, and bit-equality with the cp.async mode (the
same bytes reach the same shared-memory tile; only the copy differs)."""
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
    lib = build_library()
    yield lib
    lib.set_attn_gather(0)


def np64(t):
    return t.detach().double().cpu().numpy()


def _close(got, ref):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    assert err.max() <= ATT_MAX, f"max abs err {err.max():.3e}"
    assert err.mean() <= ATT_MEAN, f"mean abs err {err.mean():.3e}"


def _both_modes(lcsa, *args):
    outs = []
    for mode in (1, 0):
        lcsa.set_attn_gather(mode)
        try:
            outs.append(lcsa.csa_sparse_attn(*args, return_lse=True))
        finally:
            lcsa.set_attn_gather(0)
    return outs


@pytest.mark.parametrize("B,W,k,Tq,Nc,q_pos0,unit", [
    (2, 128, 256, 40, 700, 2700, True),      # layer shapes
    (2, 128, 256, 40, 700, 2700, False),     # spec scale
    (2, 128, 2048, 9, 3000, 9000, True),     # full k
    (2, 100, 100, 20, 900, 3000, True),      # odd W and k: ragged last tile and four-row groups
    (1, 128, 2048, 40, 700, 0, True),        # early rows: few visible entries, key-range splits, empty items
    (2, 128, 3000, 4, 5000, 19000, True),    # k > 2048: forced key-range splits
    (2, 128, 256, 160, 700, 2700, True),     # >= 296 rows: no split
])
def test_gather4_parity_and_equal_to_cp_async(lcsa, B, W, k, Tq, Nc, q_pos0, unit):
    H, D, R, m = 64, 512, 64, 4
    x = gen.make_attn_inputs(B, Tq, H, D, Nc, q_pos0 + Tq, "bf16", seed=151, device=DEV, unit_scale=unit,
                             with_sink=True)
    nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    idx = gen.make_topk_idx(B, Tq, k, nv, seed=152, device=DEV)
    args = (x["q"], x["ckv"], idx, x["kv"], x["sink"], q_pos0, 0, m, W, R)
    (o4, l4), (oc, lc) = _both_modes(lcsa, *args)
    torch.cuda.synchronize()
    assert lcsa.get_device_status() == 0
    assert torch.equal(o4, oc) and torch.equal(l4, lc)
    ref, ref_lse = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), idx.cpu().numpy(), np64(x["kv"]), q_pos0, 0, m,
                                     W, x["sink"].double().cpu().numpy(), R)
    _close(np64(o4).reshape(ref.shape), ref)
    np.testing.assert_allclose(np64(l4).reshape(ref_lse.shape), ref_lse, atol=2e-3)


def test_gather4_decode_slots(lcsa):
    """Decode: one query per sequence, Tq * k < Nc, so the rotary slices are
    rotated per (query, slot) and gathered by slot; window ring kv_pos0 = t-W+1."""
    B, H, D, R, m, W, k, Nc = 3, 64, 512, 64, 4, 128, 512, 4000
    t = 4 * Nc
    x = gen.make_attn_inputs(B, 1, H, D, Nc, W, "bf16", seed=153, device=DEV, unit_scale=True, with_sink=True)
    idx = gen.make_topk_idx(B, 1, k, [Nc], seed=154, device=DEV)
    args = (x["q"], x["ckv"], idx, x["kv"], x["sink"], t, t - W + 1, m, W, R)
    (o4, l4), (oc, lc) = _both_modes(lcsa, *args)
    assert torch.equal(o4, oc) and torch.equal(l4, lc)
    ref, _ = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), idx.cpu().numpy(), np64(x["kv"]), t, t - W + 1, m, W,
                               x["sink"].double().cpu().numpy(), R)
    _close(np64(o4).reshape(ref.shape), ref)


def test_gather4_bad_index_is_skipped_and_flagged(lcsa):
    """An index >= Nc reads a row past the end of the entry tensor (zeros)
    and leaves the tile's row mask; the status reports LCSA_DEV_BAD_INDEX."""
    B, H, D, R, m, W, k, Tq, Nc, q_pos0 = 1, 64, 512, 64, 4, 16, 64, 3, 500, 2400
    x = gen.make_attn_inputs(B, Tq, H, D, Nc, q_pos0 + Tq, "bf16", seed=155, device=DEV, unit_scale=True,
                             with_sink=True)
    nv = [O.n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    idx = gen.make_topk_idx(B, Tq, k, nv, seed=156, device=DEV)
    bad = idx.clone()
    bad[0, 1, 5] = Nc + 7                              # a slot inside a four-row group
    bad[0, 2, :] = Nc                                  # every slot of row 2
    assert lcsa.get_device_status() == 0
    lcsa.set_attn_gather(1)
    try:
        out = lcsa.csa_sparse_attn(x["q"], x["ckv"], bad, x["kv"], x["sink"], q_pos0, 0, m, W, R)
        assert lcsa.get_device_status() == 2
        assert lcsa.get_device_status() == 0
    finally:
        lcsa.set_attn_gather(0)
    sel = bad.cpu().numpy().copy()
    sel[sel >= Nc] = -1
    ref, _ = O.csa_sparse_attn(np64(x["q"]), np64(x["ckv"]), sel, np64(x["kv"]), q_pos0, 0, m, W,
                               x["sink"].double().cpu().numpy(), R)
    _close(np64(out).reshape(ref.shape), ref)
