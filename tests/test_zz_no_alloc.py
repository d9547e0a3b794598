"""lcsa_indexer_topk_noalloc: the indexer + top-k call for callers that cannot
allocate device memory (it runs on a fixed scratch array inside the library
instead of a caller workspace).  Called through the C ABI and compared with
lcsa_indexer_topk on the same inputs, twice in a row, so that a second call
that sees the first call's leftovers in the shared scratch is covered too.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from workloads import gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lcsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from conftest import build_library
    return build_library()


def _args(lcsa, x, q_pos0, m, k, idx_out):
    B, Tq, H_I, D_I = x["q_idx"].shape
    return lcsa.IndexerArgs(x["q_idx"].data_ptr(), x["w"].data_ptr(), x["k_idx"].data_ptr(), B, Tq,
                            x["k_idx"].shape[1], H_I, D_I, lcsa._dt(x["q_idx"]), q_pos0, m, k,
                            idx_out.data_ptr(), None)


@pytest.mark.parametrize("dtype,H_I,D_I,B,Tq,Nc,q_pos0,k", [
    # tensor-core path; 40000 entries -> ~200 score rows per scratch chunk, so 600 rows take 3 chunks
    ("bf16", 64, 128, 2, 300, 40000, 160000, 2048),
    # CUDA-core path (other shapes), rows shorter than k
    ("fp32", 2, 32, 1, 257, 300, 1000, 64),
])
def test_noalloc_matches_workspace_call(lcsa, dtype, H_I, D_I, B, Tq, Nc, q_pos0, k):
    m = 4
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((301, 302)):          # two calls in a row, different inputs
        x = gen.make_indexer_inputs(B, Tq, Nc, H_I, D_I, dtype, seed=seed, device="cuda")
        ref = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
        got = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
        a_ref = _args(lcsa, x, q_pos0, m, k, ref)
        need = lcsa.lib.lcsa_indexer_topk_workspace(ctypes.byref(a_ref))
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        assert lcsa.lib.lcsa_indexer_topk(ctypes.byref(a_ref), ctypes.c_void_p(ws.data_ptr()), need, stream) == 0
        a_got = _args(lcsa, x, q_pos0, m, k, got)
        assert lcsa.lib.lcsa_indexer_topk_noalloc(ctypes.byref(a_got), stream) == 0, f"call {call}"
        torch.cuda.synchronize()
        # identical kernels on identical scores: the index sets agree exactly
        np.testing.assert_array_equal(got.cpu().numpy(), ref.cpu().numpy())
    assert lcsa.get_device_status() == 0


def test_noalloc_rejects_rows_beyond_scratch(lcsa):
    x = gen.make_indexer_inputs(1, 4, 16, 64, 128, "bf16", seed=303, device="cuda")
    idx = torch.empty((1, 4, 16), dtype=torch.int32, device="cuda")
    a = _args(lcsa, x, 0, 4, 16, idx)
    a.Nc = 8388545                                     # one score row no longer fits 32 MiB
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lcsa.lib.lcsa_indexer_topk_noalloc(ctypes.byref(a), stream) == 3   # LCSA_ERR_WORKSPACE
