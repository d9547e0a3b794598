"""C-ABI checks that need no GPU: the library loads, exports every function
include/lcsa.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lcsa():
    from conftest import build_library
    return build_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "lcsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lcsa_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["lcsa_csa_compress", "lcsa_hca_compress", "lcsa_indexer_topk", "lcsa_topk_from_scores",
              "lcsa_csa_sparse_attn", "lcsa_hca_dense_attn", "lcsa_get_device_status"]:
        assert n in names


def test_library_exports_every_declared_symbol(lcsa):
    for n in _declared():
        assert hasattr(lcsa.lib, n), n
    assert sorted(lcsa.EXPORTED) == sorted(_declared())


def test_version_and_status_strings(lcsa):
    assert "sm_100a" in lcsa.version()
    for s in range(6):
        assert lcsa.lib.lcsa_status_string(s)


def test_struct_layouts_match_header(lcsa, tmp_path):
    """The ctypes mirrors have the C structs' size and field offsets (gcc)."""
    import subprocess
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "lcsa.h"', 'int main(void){']
    structs = (("lcsa_indexer_args", lcsa.IndexerArgs), ("lcsa_attn_args", lcsa.AttnArgs),
               ("lcsa_indexer_mxfp4_args", lcsa.IndexerMxfp4Args), ("lcsa_out_proj_args", lcsa.OutProjArgs),
               ("lcsa_fp8_entries", lcsa.Fp8Entries))
    for cname, py in structs:
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0;}")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines())
    for cname, py in structs:
        assert int(got[cname]) == ctypes.sizeof(py)
        for f, _ in py._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(py, f).offset, (cname, f)


def test_invalid_arguments_rejected_without_launch(lcsa):
    L = lcsa.lib
    # null pointers with non-empty sizes
    assert L.lcsa_csa_compress(None, None, 1, 1, 64, 512, 4, lcsa.LCSA_BF16, None, 0.0, None, lcsa.LCSA_BF16,
                               None) == 1
    # misaligned pointer (odd address) is refused before touching it
    assert L.lcsa_hca_compress(ctypes.c_void_p(0x1001), ctypes.c_void_p(0x2000), 1, 1, 256, 512, 128,
                               lcsa.LCSA_BF16, None, 0.0, ctypes.c_void_p(0x3000), lcsa.LCSA_BF16, None) == 1
    # D not a multiple of the 16-byte vector
    assert L.lcsa_csa_compress(ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), 1, 1, 64, 12, 4,
                               lcsa.LCSA_BF16, None, 0.0, ctypes.c_void_p(0x3000), lcsa.LCSA_BF16, None) == 1
    # bad k
    assert L.lcsa_topk_from_scores(ctypes.c_void_p(0x1000), 4, 16, 16, None, 0, ctypes.c_void_p(0x2000), None, 0,
                                   None) == 1
    # ld < n_cols
    assert L.lcsa_topk_from_scores(ctypes.c_void_p(0x1000), 4, 16, 8, None, 4, ctypes.c_void_p(0x2000), None, 0,
                                   None) == 1
    a = lcsa.AttnArgs()
    a.B, a.Tq, a.H, a.D, a.R, a.Nc, a.k, a.Tkv, a.m, a.W = 1, 1, 64, 512, 63, 8, 8, 8, 4, 8
    a.dtype = a.out_dtype = lcsa.LCSA_BF16
    assert L.lcsa_csa_sparse_attn(ctypes.byref(a), None, 0, None) == 1      # odd R
    a.R = 64
    assert L.lcsa_csa_sparse_attn(ctypes.byref(a), None, 0, None) == 1      # null q/out
    ia = lcsa.IndexerArgs()
    ia.B, ia.Tq, ia.Nc, ia.H_I, ia.D_I, ia.m, ia.k = 1, 4, 8, 64, 128, 0, 8
    assert L.lcsa_indexer_topk(ctypes.byref(ia), None, 0, None) == 1         # m = 0


def test_compress_entries_checks_windows(lcsa):
    """Incremental compression: windows must stay inside the raw-row buffer
    and entries inside the cache; checked before any device work."""
    L = lcsa.lib
    kv, g, c = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000)
    bf = lcsa.LCSA_BF16
    # buffer positions [120, 248): CSA entry 61 pools [240, 248) -> fine; entry 29 pools [112, 120) -> outside
    args = lambda j0, n, rows, pos0=120, window=8: (kv, g, 1, 1, 128, 512, pos0, 4, window, j0, n, bf, None, 0.0, c,
                                                    rows, bf, None)
    assert L.lcsa_compress_entries(*args(29, 1, 64)) == 1              # window starts before the buffer
    assert L.lcsa_compress_entries(*args(62, 1, 64)) == 1              # window ends after the buffer
    assert L.lcsa_compress_entries(*args(61, 1, 61)) == 1              # entry beyond the cache
    assert L.lcsa_compress_entries(*args(-1, 1, 64)) == 1              # negative first entry
    assert L.lcsa_compress_entries(*args(61, 1, 64, window=0)) == 1    # empty window
    assert L.lcsa_compress_entries(*args(61, 0, 64)) == 0              # nothing to do
    if not torch.cuda.is_available():
        assert L.lcsa_compress_entries(*args(61, 1, 64)) == 4          # valid, but no device: no CPU path
        assert L.lcsa_compress_entries(*args(31, 30, 64)) == 4         # entries 31..60 pool [120, 244)


def test_mxfp4_calls_check_arguments(lcsa):
    L = lcsa.lib
    x, c, sc = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000)
    assert L.lcsa_quantize_mxfp4(x, 4, 48, lcsa.LCSA_BF16, c, sc, None) == 1       # cols not a multiple of 32
    assert L.lcsa_quantize_mxfp4(None, 4, 64, lcsa.LCSA_BF16, c, sc, None) == 1    # null input
    assert L.lcsa_quantize_mxfp4(ctypes.c_void_p(0x1001), 4, 64, lcsa.LCSA_BF16, c, sc, None) == 1   # misaligned
    assert L.lcsa_quantize_mxfp4(None, 0, 64, lcsa.LCSA_BF16, None, None, None) == 0  # nothing to do
    a = lcsa.IndexerMxfp4Args()
    a.q_idx, a.w, a.k_codes, a.k_scales, a.idx_out = 0x1000, 0x2000, 0x3000, 0x4000, 0x5000
    a.B, a.Tq, a.Nc, a.H_I, a.D_I, a.m, a.k = 1, 4, 8, 64, 64, 4, 8
    assert L.lcsa_indexer_topk_mxfp4(ctypes.byref(a), None, 0, None) == 2         # D_I = 64: unsupported
    a.D_I = 128
    a.k_scales = 0x4002
    assert L.lcsa_indexer_topk_mxfp4(ctypes.byref(a), None, 0, None) == 1         # misaligned scales
    a.k_scales, a.m = 0x4000, 0
    assert L.lcsa_indexer_topk_mxfp4(ctypes.byref(a), None, 0, None) == 1         # m = 0
    a.m = 4
    assert L.lcsa_indexer_topk_mxfp4_workspace(ctypes.byref(a)) > L.lcsa_indexer_topk_workspace(
        ctypes.byref(lcsa.IndexerArgs(None, None, None, 1, 4, 8, 64, 128, lcsa.LCSA_BF16, 0, 4, 8, None, None)))
    if not torch.cuda.is_available():
        ws = ctypes.c_void_p(0x10000)
        assert L.lcsa_indexer_topk_mxfp4(ctypes.byref(a), ws, 1 << 20, None) == 4   # no device: no CPU path


def test_grouped_out_proj_checks_arguments(lcsa):
    L = lcsa.lib
    P = lambda **kw: lcsa.OutProjArgs(**{"o": 0x1000, "w_group": 0x2000, "w_out": 0x3000, "y": 0x4000, "T": 16,
                                        "n_h": 64, "c": 512, "g": 8, "d_g": 1024, "d": 4096, **kw})
    ws = ctypes.c_void_p(0x10000)
    assert L.lcsa_grouped_out_proj(ctypes.byref(P(g=7)), ws, 1 << 30, None) == 1        # g does not divide n_h
    assert L.lcsa_grouped_out_proj(ctypes.byref(P(c=36)), ws, 1 << 30, None) == 1       # K = 288, not a multiple of 64
    assert L.lcsa_grouped_out_proj(ctypes.byref(P(d=100)), ws, 1 << 30, None) == 1      # d not a multiple of 8
    assert L.lcsa_grouped_out_proj(ctypes.byref(P(y=0x4008)), ws, 1 << 30, None) == 1   # misaligned output
    assert L.lcsa_grouped_out_proj(ctypes.byref(P()), ws, 64, None) == 3                # workspace too small
    assert L.lcsa_grouped_out_proj(ctypes.byref(P(T=0)), None, 0, None) == 0            # nothing to do
    assert L.lcsa_grouped_out_proj_workspace(ctypes.byref(P())) == 16 * 8 * 1024 * 2
    if not torch.cuda.is_available():
        assert L.lcsa_grouped_out_proj(ctypes.byref(P()), ws, 1 << 30, None) == 4       # no device: no CPU path


def test_empty_problems_are_noops(lcsa):
    L = lcsa.lib
    # T < m: no entries, nothing to do, no device needed
    assert L.lcsa_csa_compress(None, None, 1, 1, 3, 512, 4, lcsa.LCSA_BF16, None, 0.0, None, lcsa.LCSA_BF16,
                               None) == 0
    assert L.lcsa_topk_from_scores(None, 0, 16, 16, None, 4, None, None, 0, None) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device behaviour")
def test_no_cpu_fallback(lcsa):
    """Without a CUDA device a valid compute call fails loudly (no CPU path)."""
    L = lcsa.lib
    st = L.lcsa_csa_compress(ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), 1, 1, 64, 512, 4,
                             lcsa.LCSA_BF16, None, 0.0, ctypes.c_void_p(0x3000), lcsa.LCSA_BF16, None)
    assert st == 4


def test_workspace_queries(lcsa):
    q = torch.empty((1, 4096, 64, 128), dtype=torch.bfloat16)
    k = torch.empty((1, 1024, 128), dtype=torch.bfloat16)
    assert lcsa.indexer_workspace_bytes(q, k, 2048) >= 4096 * 1024 * 4


def test_noalloc_validates_like_the_workspace_call(lcsa):
    """lcsa_indexer_topk_noalloc runs lcsa_indexer_topk's argument checks first,
    so a bad argument gives the same status through both entry points, before
    anything touches a device."""
    L = lcsa.lib
    ptrs = dict(q_idx=0x1000, w=0x2000, k_idx=0x3000, idx_out=0x4000)
    base = dict(B=1, Tq=4, Nc=8, H_I=64, D_I=128, dtype=lcsa.LCSA_BF16, q_pos0=0, m=4, k=8)
    cases = [dict(Nc=-1), dict(m=0), dict(k=0), dict(q_pos0=-5), dict(idx_out=0x4004), dict(w=0)]
    for c in cases:
        a = lcsa.IndexerArgs(**{**ptrs, **base, **c})
        assert L.lcsa_indexer_topk(ctypes.byref(a), None, 0, None) == 1, c
        assert L.lcsa_indexer_topk_noalloc(ctypes.byref(a), None) == 1, c
    # 8,388,544 scores of one row fill the 32 MiB scratch exactly: with k = 2048 the row
    # takes the single-phase top-k (more than 16 chunks of 32768) and fits; with k = 64
    # its two-phase top-k scratch (256 chunks x 64 winners) does not; one more column never fits
    a = lcsa.IndexerArgs(**{**ptrs, **base, "Nc": 8388544, "k": 64})
    assert L.lcsa_indexer_topk_noalloc(ctypes.byref(a), None) == 3
    a.k, a.Nc = 2048, 8388545
    assert L.lcsa_indexer_topk_noalloc(ctypes.byref(a), None) == 3
    if not torch.cuda.is_available():
        a.Nc = 8388544
        assert L.lcsa_indexer_topk_noalloc(ctypes.byref(a), None) == 4     # fits; no device: no CPU path


def test_fp8_cache_calls_check_arguments(lcsa):
    L = lcsa.lib
    x, c, sc, r = (ctypes.c_void_p(v) for v in (0x1000, 0x2000, 0x3000, 0x4000))
    assert L.lcsa_quantize_entries_fp8(x, 4, 512, 63, lcsa.LCSA_BF16, c, sc, r, None) == 1     # odd R
    assert L.lcsa_quantize_entries_fp8(x, 4, 512, 512, lcsa.LCSA_BF16, c, sc, r, None) == 1    # R = D
    assert L.lcsa_quantize_entries_fp8(None, 4, 512, 64, lcsa.LCSA_BF16, c, sc, r, None) == 1  # null input
    assert L.lcsa_quantize_entries_fp8(ctypes.c_void_p(0x1001), 4, 512, 64, lcsa.LCSA_BF16, c, sc, r, None) == 1
    assert L.lcsa_quantize_entries_fp8(None, 0, 512, 64, lcsa.LCSA_BF16, None, None, None, None) == 0
    a = lcsa.AttnArgs()
    a.q, a.out, a.kv, a.idx = 0x10000, 0x20000, 0x30000, 0x40000
    a.B, a.Tq, a.H, a.D, a.R, a.Nc, a.k, a.Tkv, a.m, a.W = 1, 1, 64, 512, 64, 8, 8, 8, 4, 8
    a.dtype = a.out_dtype = lcsa.LCSA_BF16
    e = lcsa.Fp8Entries(0x50000, 0x60000, 0x70000)
    assert L.lcsa_csa_sparse_attn_fp8(ctypes.byref(a), None, None, 0, None) == 1          # no cache
    e.codes = 0x50008
    assert L.lcsa_csa_sparse_attn_fp8(ctypes.byref(a), ctypes.byref(e), None, 0, None) == 1   # misaligned codes
    e.codes = 0x50000
    a.H = 16
    assert L.lcsa_hca_dense_attn_fp8(ctypes.byref(a), ctypes.byref(e), None, 0, None) == 2    # not the layer shape
    a.H = 64
    if not torch.cuda.is_available():
        ws = ctypes.c_void_p(0x100000)
        assert L.lcsa_hca_dense_attn_fp8(ctypes.byref(a), ctypes.byref(e), ws, 1 << 30, None) == 4   # no CPU path


def test_attn_gather_mode_argument(lcsa):
    """The CSA row-staging switch takes 0 (cp.async) or 1 (TMA gather) only."""
    L = lcsa.lib
    assert L.lcsa_set_attn_gather(2) == 1 and L.lcsa_set_attn_gather(-1) == 1
    assert L.lcsa_set_attn_gather(1) == 0
    assert L.lcsa_set_attn_gather(0) == 0


def test_fp4_mma_mode_argument(lcsa):
    """The MXFP4 key path switch takes 0 (E4M3 staging) or 1 (block-scaled MMA) only."""
    L = lcsa.lib
    assert L.lcsa_set_fp4_mma(2) == 1 and L.lcsa_set_fp4_mma(-1) == 1
    assert L.lcsa_set_fp4_mma(0) == 0
    assert L.lcsa_set_fp4_mma(1) == 0
