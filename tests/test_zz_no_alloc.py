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


_CONTEXT_CHILD = r'''
import ctypes, sys
import numpy as np
from ctypes import byref, c_int, c_size_t, c_uint64, c_void_p

cu = ctypes.CDLL("libcuda.so.1")
lib = ctypes.CDLL(sys.argv[1])
sys.path.insert(0, sys.argv[2])
from long_context_compressed_softmax_b200 import IndexerArgs   # ctypes mirror only (needs torch, no GPU work)


def ok(r, what):
    if r != 0:
        raise SystemExit(f"{what}: CUresult {r}")


ok(cu.cuInit(0), "cuInit")
dev = c_int()
ok(cu.cuDeviceGet(byref(dev), 0), "cuDeviceGet")
rng = np.random.default_rng(404)
B, Tq, Nc, H_I, D_I, q_pos0, m, k = 1, 96, 3000, 64, 128, 12000, 4, 256


def bf16(x):                                   # round to nearest even, as uint16 bit patterns
    u = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


host = {"q": bf16(rng.standard_normal((B, Tq, H_I, D_I)) / np.sqrt(D_I)),
        "w": (rng.standard_normal((B, Tq, H_I)) / 8).astype(np.float32),
        "k": bf16(rng.standard_normal((B, Nc, D_I)) / np.sqrt(D_I))}


def alloc(nbytes):
    p = c_uint64()
    ok(cu.cuMemAlloc_v2(byref(p), c_size_t(nbytes)), "cuMemAlloc")
    return p.value


def run_in_current_context():
    d = {}
    for name, arr in host.items():
        d[name] = alloc(arr.nbytes)
        ok(cu.cuMemcpyHtoD_v2(c_uint64(d[name]), arr.ctypes.data_as(c_void_p), c_size_t(arr.nbytes)), "HtoD")
    outs = []
    for noalloc in (False, True, True):        # the workspace call, then two scratch calls in a row
        idx = alloc(B * Tq * k * 4)
        a = IndexerArgs(d["q"], d["w"], d["k"], B, Tq, Nc, H_I, D_I, 1, q_pos0, m, k, idx, None)
        if noalloc:
            st = lib.lcsa_indexer_topk_noalloc(byref(a), None)
        else:
            lib.lcsa_indexer_topk_workspace.restype = c_size_t
            need = lib.lcsa_indexer_topk_workspace(byref(a))
            st = lib.lcsa_indexer_topk(byref(a), c_void_p(alloc(need)), c_size_t(need), None)
        if st != 0:
            raise SystemExit(f"lcsa call (noalloc={noalloc}) returned {st}")
        ok(cu.cuCtxSynchronize(), "cuCtxSynchronize")
        h = np.empty((B, Tq, k), dtype=np.int32)
        ok(cu.cuMemcpyDtoH_v2(h.ctypes.data_as(c_void_p), c_uint64(idx), c_size_t(h.nbytes)), "DtoH")
        outs.append(h)
    for h in outs[1:]:
        if not np.array_equal(h, outs[0]):
            raise SystemExit("scratch call differs from the workspace call")
    return outs[0]


primary = c_void_p()
ok(cu.cuDevicePrimaryCtxRetain(byref(primary), dev), "cuDevicePrimaryCtxRetain")
ok(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
r_primary = run_in_current_context()
other = c_void_p()
ok(cu.cuCtxCreate_v2(byref(other), 0, dev), "cuCtxCreate")          # a second context, now current
r_other = run_in_current_context()
ok(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")                   # back to the first one
r_back = run_in_current_context()
ok(cu.cuCtxDestroy_v2(other), "cuCtxDestroy")
# a reset of this process's primary context (what cudaDeviceReset does): the
# module is loaded again and the scratch array gets a new address
ok(cu.cuCtxSetCurrent(None), "cuCtxSetCurrent")
ok(cu.cuDevicePrimaryCtxRelease_v2(dev), "cuDevicePrimaryCtxRelease")
ok(cu.cuDevicePrimaryCtxReset_v2(dev), "cuDevicePrimaryCtxReset")
fresh = c_void_p()
ok(cu.cuDevicePrimaryCtxRetain(byref(fresh), dev), "cuDevicePrimaryCtxRetain")
ok(cu.cuCtxSetCurrent(fresh), "cuCtxSetCurrent")
r_reset = run_in_current_context()
if not (np.array_equal(r_primary, r_other) and np.array_equal(r_primary, r_back)
        and np.array_equal(r_primary, r_reset)):
    raise SystemExit("results differ between contexts")
print("contexts ok")
'''


def test_noalloc_in_two_contexts(lcsa, tmp_path):
    """The scratch array's device address belongs to a context.  A caller that
    switches between the primary context and a context of its own (driver API),
    and then resets the primary context (as cudaDeviceReset does), gets correct
    results each time, every call matching the workspace call.  Runs
    in a child process that uses only the driver API, so this process's
    contexts are not touched."""
    import os
    import subprocess
    import sys
    child = tmp_path / "contexts_child.py"
    child.write_text(_CONTEXT_CHILD)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, str(child), lcsa.LIB_PATH, root], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "contexts ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
