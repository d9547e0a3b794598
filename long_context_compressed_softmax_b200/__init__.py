"""Python binding of liblcsa (argument marshalling only).

Every call forwards raw device pointers, sizes and the current CUDA stream to
the C ABI declared in include/lcsa.h; all computation runs in the library's
sm_100a kernels.  PyTorch is used for device memory and streams.  There is no
fallback: if liblcsa.so is missing, importing this package fails.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblcsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"liblcsa.so not found at {LIB_PATH}; build it with "
        "`python -m long_context_compressed_softmax_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

LCSA_FP32, LCSA_BF16 = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported combination", 3: "workspace missing or too small",
           4: "CUDA error", 5: "device reported an error"}

EXPORTED = [
    "lcsa_version", "lcsa_status_string", "lcsa_get_device_status", "lcsa_kernel_launches",
    "lcsa_csa_compress", "lcsa_hca_compress",
    "lcsa_compress_entries",
    "lcsa_topk_workspace", "lcsa_topk_from_scores",
    "lcsa_indexer_topk_workspace", "lcsa_indexer_topk", "lcsa_indexer_uses_tensor_cores",
    "lcsa_indexer_topk_noalloc",
    "lcsa_quantize_mxfp4", "lcsa_indexer_topk_mxfp4_workspace", "lcsa_indexer_topk_mxfp4",
    "lcsa_grouped_out_proj_workspace", "lcsa_grouped_out_proj",
    "lcsa_attn_workspace", "lcsa_csa_sparse_attn", "lcsa_hca_dense_attn", "lcsa_attn_uses_tensor_cores",
    "lcsa_quantize_entries_fp8", "lcsa_csa_sparse_attn_fp8", "lcsa_hca_dense_attn_fp8",
    "lcsa_set_wait_limit_ns", "lcsa_test_withhold_stage", "lcsa_set_attn_gather", "lcsa_set_fp4_mma",
]


class LcsaError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = int(status)
        super().__init__(f"{what}: {_STATUS.get(self.status, self.status)} ({self.status})")


class IndexerArgs(ctypes.Structure):
    _fields_ = [
        ("q_idx", ctypes.c_void_p), ("w", ctypes.c_void_p), ("k_idx", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Tq", ctypes.c_int), ("Nc", ctypes.c_int), ("H_I", ctypes.c_int),
        ("D_I", ctypes.c_int), ("dtype", ctypes.c_int), ("q_pos0", ctypes.c_int64), ("m", ctypes.c_int),
        ("k", ctypes.c_int), ("idx_out", ctypes.c_void_p), ("scores_out", ctypes.c_void_p),
    ]


class IndexerMxfp4Args(ctypes.Structure):
    _fields_ = [
        ("q_idx", ctypes.c_void_p), ("w", ctypes.c_void_p), ("k_codes", ctypes.c_void_p),
        ("k_scales", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Tq", ctypes.c_int), ("Nc", ctypes.c_int), ("H_I", ctypes.c_int),
        ("D_I", ctypes.c_int), ("q_pos0", ctypes.c_int64), ("m", ctypes.c_int), ("k", ctypes.c_int),
        ("idx_out", ctypes.c_void_p), ("scores_out", ctypes.c_void_p),
    ]


class OutProjArgs(ctypes.Structure):
    _fields_ = [
        ("o", ctypes.c_void_p), ("w_group", ctypes.c_void_p), ("w_out", ctypes.c_void_p), ("y", ctypes.c_void_p),
        ("T", ctypes.c_int), ("n_h", ctypes.c_int), ("c", ctypes.c_int), ("g", ctypes.c_int), ("d_g", ctypes.c_int),
        ("d", ctypes.c_int),
    ]


class AttnArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("ckv", ctypes.c_void_p), ("idx", ctypes.c_void_p), ("kv", ctypes.c_void_p),
        ("sink", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Tq", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int), ("R", ctypes.c_int),
        ("Nc", ctypes.c_int), ("k", ctypes.c_int), ("Tkv", ctypes.c_int),
        ("q_pos0", ctypes.c_int64), ("kv_pos0", ctypes.c_int64),
        ("m", ctypes.c_int), ("W", ctypes.c_int), ("softmax_scale", ctypes.c_float), ("rope_base", ctypes.c_float),
        ("dtype", ctypes.c_int), ("out", ctypes.c_void_p), ("out_dtype", ctypes.c_int), ("lse", ctypes.c_void_p),
    ]


class Fp8Entries(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rope", ctypes.c_void_p)]


_vp, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_sig = {
    "lcsa_version": (ctypes.c_char_p, []),
    "lcsa_status_string": (ctypes.c_char_p, [_i]),
    "lcsa_kernel_launches": (ctypes.c_uint64, []),
    "lcsa_get_device_status": (_i, [_vp, ctypes.POINTER(_i)]),
    "lcsa_csa_compress": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _i, _vp]),
    "lcsa_hca_compress": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _vp, _i, _vp]),
    "lcsa_compress_entries": (_i, [_vp, _vp, _i, _i, _i, _i, _i64, _i, _i, _i64, _i, _i, _vp, ctypes.c_float, _vp,
                                   _i64, _i, _vp]),
    "lcsa_topk_workspace": (_sz, [_i, _i, _i]),
    "lcsa_topk_from_scores": (_i, [_vp, _i, _i, _i64, _vp, _i, _vp, _vp, _sz, _vp]),
    "lcsa_indexer_topk_workspace": (_sz, [ctypes.POINTER(IndexerArgs)]),
    "lcsa_indexer_topk": (_i, [ctypes.POINTER(IndexerArgs), _vp, _sz, _vp]),
    "lcsa_indexer_uses_tensor_cores": (_i, [ctypes.POINTER(IndexerArgs)]),
    "lcsa_indexer_topk_noalloc": (_i, [ctypes.POINTER(IndexerArgs), _vp]),
    "lcsa_quantize_mxfp4": (_i, [_vp, _i64, _i, _i, _vp, _vp, _vp]),
    "lcsa_indexer_topk_mxfp4_workspace": (_sz, [ctypes.POINTER(IndexerMxfp4Args)]),
    "lcsa_indexer_topk_mxfp4": (_i, [ctypes.POINTER(IndexerMxfp4Args), _vp, _sz, _vp]),
    "lcsa_grouped_out_proj_workspace": (_sz, [ctypes.POINTER(OutProjArgs)]),
    "lcsa_grouped_out_proj": (_i, [ctypes.POINTER(OutProjArgs), _vp, _sz, _vp]),
    "lcsa_attn_workspace": (_sz, [ctypes.POINTER(AttnArgs), _i]),
    "lcsa_csa_sparse_attn": (_i, [ctypes.POINTER(AttnArgs), _vp, _sz, _vp]),
    "lcsa_hca_dense_attn": (_i, [ctypes.POINTER(AttnArgs), _vp, _sz, _vp]),
    "lcsa_attn_uses_tensor_cores": (_i, [ctypes.POINTER(AttnArgs)]),
    "lcsa_quantize_entries_fp8": (_i, [_vp, _i64, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "lcsa_set_wait_limit_ns": (_i, [ctypes.c_uint64]),
    "lcsa_test_withhold_stage": (None, [_i]),
    "lcsa_set_attn_gather": (_i, [_i]),
    "lcsa_set_fp4_mma": (_i, [_i]),
    "lcsa_csa_sparse_attn_fp8": (_i, [ctypes.POINTER(AttnArgs), ctypes.POINTER(Fp8Entries), _vp, _sz, _vp]),
    "lcsa_hca_dense_attn_fp8": (_i, [ctypes.POINTER(AttnArgs), ctypes.POINTER(Fp8Entries), _vp, _sz, _vp]),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

lib = _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LCSA_BF16
    if t.dtype == torch.float32:
        return LCSA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _tdt(code: int) -> torch.dtype:
    return torch.bfloat16 if code == LCSA_BF16 else torch.float32


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(status, what):
    if status != 0:
        raise LcsaError(status, what)


def _need_contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def version() -> str:
    return _lib.lcsa_version().decode()


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(_lib.lcsa_kernel_launches())


def set_wait_limit_ns(ns: int) -> None:
    """Limit of the kernels' bounded waits on the current device (0 = the 2 s default)."""
    _check(_lib.lcsa_set_wait_limit_ns(int(ns)), "set_wait_limit_ns")


def set_attn_gather(mode: int) -> None:
    """CSA row staging on BF16 entries: 0 = cp.async (default), 1 = TMA tile::gather4."""
    _check(_lib.lcsa_set_attn_gather(int(mode)), "set_attn_gather")


def set_fp4_mma(mode: int) -> None:
    """MXFP4 indexer keys: 0 = E4M3 staging (default), 1 = block-scaled MMA on the codes for 1-2 row calls."""
    _check(_lib.lcsa_set_fp4_mma(int(mode)), "set_fp4_mma")


def get_device_status() -> int:
    code = ctypes.c_int(0)
    st = _lib.lcsa_get_device_status(_stream(), ctypes.byref(code))
    if st not in (0, 5):
        raise LcsaError(st, "lcsa_get_device_status")
    return code.value


# ----------------------------------------------------------------- compress
def _compress(fn, name, kv, gate, m, out_dtype, rms_weight, rms_eps, out):
    _need_contig(kv, gate, rms_weight)
    B, T, D = kv.shape
    per_channel = 1 if gate.dim() == 3 else 0
    odt = _dt(kv) if out_dtype is None else (LCSA_BF16 if out_dtype == torch.bfloat16 else LCSA_FP32)
    if out is None:
        out = torch.empty((B, T // m, D), dtype=_tdt(odt), device=kv.device)
    st = fn(_p(kv), _p(gate), per_channel, B, T, D, m, _dt(kv), _p(rms_weight), float(rms_eps), _p(out), odt,
            _stream(kv.device))
    _check(st, name)
    return out


def csa_compress(kv, gate, m=4, out_dtype=None, rms_weight=None, rms_eps=1e-6, out=None):
    """kv [B,T,D], gate [B,T,D] or [B,T] -> [B,T//m,D] (window 2m, stride m)."""
    return _compress(_lib.lcsa_csa_compress, "csa_compress", kv, gate, m, out_dtype, rms_weight, rms_eps, out)


def hca_compress(kv, gate, m=128, out_dtype=None, rms_weight=None, rms_eps=1e-6, out=None):
    """kv [B,T,D], gate [B,T,D] or [B,T] -> [B,T//m,D] (non-overlapping blocks)."""
    return _compress(_lib.lcsa_hca_compress, "hca_compress", kv, gate, m, out_dtype, rms_weight, rms_eps, out)


# ----------------------------------------------------------------- top-k
def compress_entries(kv, gate, kv_pos0, m, window, j0, n_entries, cache, rms_weight=None, rms_eps=1e-6):
    """Entries j0 .. j0+n_entries-1 of a compressed cache from a buffer of raw
    rows: kv [B,Tkv,D] holds positions kv_pos0 .. kv_pos0+Tkv-1, gate
    [B,Tkv,D] or [B,Tkv]; window 2m (CSA) or m (HCA); written into cache
    [B,cache_rows,D] at rows j (incremental decode compression)."""
    _need_contig(kv, gate, cache)
    B, Tkv, D = kv.shape
    per_channel = 1 if gate.dim() == 3 else 0
    st = _lib.lcsa_compress_entries(_p(kv), _p(gate), per_channel, B, Tkv, D, int(kv_pos0), m, window, int(j0),
                                    n_entries, _dt(kv), _p(rms_weight), float(rms_eps), _p(cache), cache.shape[1],
                                    _dt(cache), _stream(kv.device))
    _check(st, "compress_entries")
    return cache


def topk_workspace_bytes(rows, n_cols, k):
    """Scratch that lets rows longer than 32768 columns take the two-phase path."""
    return int(_lib.lcsa_topk_workspace(rows, n_cols, k))


def topk_from_scores(scores, k, n_valid=None, out=None, workspace=None):
    """scores [rows, n_cols] fp32 (row stride may exceed n_cols) -> idx [rows, k] int32.

    workspace: None allocates the scratch of topk_workspace_bytes; a uint8
    tensor is used as is; False passes none (long rows then use the
    single-phase kernel)."""
    rows, n_cols = scores.shape
    if scores.stride(1) != 1:
        raise ValueError("scores rows must be contiguous")
    if out is None:
        out = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    if workspace is None:
        nbytes = topk_workspace_bytes(rows, n_cols, k)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=scores.device) if nbytes else False
    ws_ptr, ws_bytes = (None, 0) if workspace is False else (_p(workspace), workspace.numel())
    st = _lib.lcsa_topk_from_scores(_p(scores), rows, n_cols, scores.stride(0), _p(n_valid), k, _p(out), ws_ptr,
                                    ws_bytes, _stream(scores.device))
    _check(st, "topk_from_scores")
    return out


# ----------------------------------------------------------------- indexer
def _indexer_args(q_idx, w, k_idx, q_pos0, m, k, idx_out, scores_out):
    B, Tq, H_I, D_I = q_idx.shape
    return IndexerArgs(_p(q_idx), _p(w), _p(k_idx), B, Tq, k_idx.shape[1], H_I, D_I, _dt(q_idx), int(q_pos0), m, k,
                       _p(idx_out), _p(scores_out))


def indexer_workspace_bytes(q_idx, k_idx, k):
    B, Tq, H_I, D_I = q_idx.shape
    a = IndexerArgs(None, None, None, B, Tq, k_idx.shape[1], H_I, D_I, _dt(q_idx), 0, 1, k, None, None)
    return int(_lib.lcsa_indexer_topk_workspace(ctypes.byref(a)))


def indexer_uses_tensor_cores(q_idx, k_idx, k):
    B, Tq, H_I, D_I = q_idx.shape
    a = IndexerArgs(None, None, None, B, Tq, k_idx.shape[1], H_I, D_I, _dt(q_idx), 0, 1, k, None, None)
    return bool(_lib.lcsa_indexer_uses_tensor_cores(ctypes.byref(a)))


def indexer_topk(q_idx, w, k_idx, q_pos0, m, k, return_scores=False, workspace=None, idx_out=None):
    """q_idx [B,Tq,H_I,D_I], w [B,Tq,H_I] fp32, k_idx [B,Nc,D_I] -> idx [B,Tq,k] int32
    (and scores [B,Tq,Nc] fp32 when return_scores)."""
    _need_contig(q_idx, w, k_idx)
    B, Tq = q_idx.shape[:2]
    Nc = k_idx.shape[1]
    dev = q_idx.device
    if idx_out is None:
        idx_out = torch.empty((B, Tq, k), dtype=torch.int32, device=dev)
    scores = torch.empty((B, Tq, Nc), dtype=torch.float32, device=dev) if return_scores else None
    a = _indexer_args(q_idx, w, k_idx, q_pos0, m, k, idx_out, scores)
    need = int(_lib.lcsa_indexer_topk_workspace(ctypes.byref(a)))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    st = _lib.lcsa_indexer_topk(ctypes.byref(a), _p(workspace), workspace.numel(), _stream(dev))
    _check(st, "indexer_topk")
    return (idx_out, scores) if return_scores else idx_out


# ----------------------------------------------------------------- FP4 indexer path
def quantize_mxfp4(x, codes=None, scales=None):
    """MXFP4 of x [..., C] (BF16 or FP32, C a multiple of 32) along the last
    axis -> (codes uint8 [..., C/2], scales uint8 [..., C/32])."""
    _need_contig(x)
    C = x.shape[-1]
    rows = x.numel() // C if C else 0
    if codes is None:
        codes = torch.empty(x.shape[:-1] + (C // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1] + (C // 32,), dtype=torch.uint8, device=x.device)
    st = _lib.lcsa_quantize_mxfp4(_p(x), rows, C, _dt(x), _p(codes), _p(scales), _stream(x.device))
    _check(st, "quantize_mxfp4")
    return codes, scales


def _indexer_mxfp4_args(q_idx, w, k_codes, k_scales, q_pos0, m, k, idx_out, scores_out):
    B, Tq, H_I, D_I = q_idx.shape
    return IndexerMxfp4Args(_p(q_idx), _p(w), _p(k_codes), _p(k_scales), B, Tq, k_codes.shape[1], H_I, D_I,
                            int(q_pos0), m, k, _p(idx_out), _p(scores_out))


def indexer_mxfp4_workspace_bytes(q_idx, k_codes, k):
    B, Tq, H_I, D_I = q_idx.shape
    a = IndexerMxfp4Args(None, None, None, None, B, Tq, k_codes.shape[1], H_I, D_I, 0, 1, k, None, None)
    return int(_lib.lcsa_indexer_topk_mxfp4_workspace(ctypes.byref(a)))


def indexer_topk_mxfp4(q_idx, w, k_codes, k_scales, q_pos0, m, k, return_scores=False, workspace=None,
                       idx_out=None):
    """FP4 QK path: q_idx [B,Tq,64,128] BF16, w [B,Tq,64] fp32, MXFP4 keys
    k_codes [B,Nc,64] / k_scales [B,Nc,4] uint8 -> idx [B,Tq,k] int32 (and
    scores [B,Tq,Nc] fp32 when return_scores)."""
    _need_contig(q_idx, w, k_codes, k_scales)
    B, Tq = q_idx.shape[:2]
    Nc = k_codes.shape[1]
    dev = q_idx.device
    if idx_out is None:
        idx_out = torch.empty((B, Tq, k), dtype=torch.int32, device=dev)
    scores = torch.empty((B, Tq, Nc), dtype=torch.float32, device=dev) if return_scores else None
    a = _indexer_mxfp4_args(q_idx, w, k_codes, k_scales, q_pos0, m, k, idx_out, scores)
    if workspace is None:       # a smaller caller workspace processes fewer rows at a time
        need = int(_lib.lcsa_indexer_topk_mxfp4_workspace(ctypes.byref(a)))
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    st = _lib.lcsa_indexer_topk_mxfp4(ctypes.byref(a), _p(workspace), workspace.numel(), _stream(dev))
    _check(st, "indexer_topk_mxfp4")
    return (idx_out, scores) if return_scores else idx_out


# ----------------------------------------------------------------- grouped output projection
def grouped_out_proj_workspace_bytes(T, g, d_g):
    a = OutProjArgs(None, None, None, None, T, g, 1, g, d_g, 8)
    return int(_lib.lcsa_grouped_out_proj_workspace(ctypes.byref(a)))


def grouped_out_proj(o, w_group, w_out, out=None, workspace=None):
    """o [T, n_h, c] BF16, w_group [g, d_g, n_h/g*c] BF16, w_out [d, g*d_g] BF16
    -> y [T, d] BF16 (per-group projection to d_g, merge projection to d)."""
    _need_contig(o, w_group, w_out)
    T, n_h, c = o.shape
    g, d_g, _ = w_group.shape
    d = w_out.shape[0]
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=o.device)
    a = OutProjArgs(_p(o), _p(w_group), _p(w_out), _p(out), T, n_h, c, g, d_g, d)
    if workspace is None:
        need = int(_lib.lcsa_grouped_out_proj_workspace(ctypes.byref(a)))
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=o.device)
    st = _lib.lcsa_grouped_out_proj(ctypes.byref(a), _p(workspace), workspace.numel(), _stream(o.device))
    _check(st, "grouped_out_proj")
    return out


# ----------------------------------------------------------------- attention
def _attn_args(q, ckv, idx, kv, sink, q_pos0, kv_pos0, m, W, R, softmax_scale, rope_base, out, lse):
    B, Tq, H, D = q.shape
    k = idx.shape[2] if idx is not None else 0
    return AttnArgs(_p(q), _p(ckv), _p(idx), _p(kv), _p(sink), B, Tq, H, D, R, ckv.shape[1], k, kv.shape[1],
                    int(q_pos0), int(kv_pos0), m, W, float(softmax_scale), float(rope_base), _dt(q), _p(out),
                    _dt(out), _p(lse))


def attn_workspace_bytes(q, ckv, idx, kv, m, W, R=64, sparse=True, q_pos0=0, kv_pos0=0):
    a = _attn_args(q, ckv, idx, kv, None, q_pos0, kv_pos0, m, W, R, 0.0, 0.0, q, None)
    return int(_lib.lcsa_attn_workspace(ctypes.byref(a), 1 if sparse else 0))


def attn_uses_tensor_cores(q, ckv, kv, R=64):
    a = _attn_args(q, ckv, None, kv, None, 0, 0, 1, 0, R, 0.0, 0.0, q, None)
    return bool(_lib.lcsa_attn_uses_tensor_cores(ctypes.byref(a)))


def _attn(fn, name, sparse, q, ckv, idx, kv, sink, q_pos0, kv_pos0, m, W, R, softmax_scale, rope_base, out_dtype,
          return_lse, workspace, out):
    _need_contig(q, ckv, idx, kv, sink)
    B, Tq, H, D = q.shape
    dev = q.device
    if out is None:
        out = torch.empty((B, Tq, H, D), dtype=out_dtype, device=dev)
    lse = torch.empty((B, Tq, H), dtype=torch.float32, device=dev) if return_lse else None
    a = _attn_args(q, ckv, idx, kv, sink, q_pos0, kv_pos0, m, W, R, softmax_scale, rope_base, out, lse)
    need = int(_lib.lcsa_attn_workspace(ctypes.byref(a), sparse))
    if need > 0 and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_n = 0 if workspace is None else workspace.numel()
    st = fn(ctypes.byref(a), _p(workspace), ws_n, _stream(dev))
    _check(st, name)
    return (out, lse) if return_lse else out


def csa_sparse_attn(q, ckv, idx, kv, sink, q_pos0, kv_pos0, m=4, W=128, R=64, softmax_scale=0.0,
                    rope_base=10000.0, out_dtype=torch.float32, return_lse=False, workspace=None, out=None):
    """CSA core attention over the selected entries idx [B,Tq,k] plus the window and sink."""
    return _attn(_lib.lcsa_csa_sparse_attn, "csa_sparse_attn", 1, q, ckv, idx, kv, sink, q_pos0, kv_pos0, m, W, R,
                 softmax_scale, rope_base, out_dtype, return_lse, workspace, out)


def hca_dense_attn(q, ckv, kv, sink, q_pos0, kv_pos0, m=128, W=128, R=64, softmax_scale=0.0, rope_base=10000.0,
                   out_dtype=torch.float32, return_lse=False, workspace=None, out=None):
    """HCA core attention over every visible entry plus the window and sink."""
    return _attn(_lib.lcsa_hca_dense_attn, "hca_dense_attn", 0, q, ckv, None, kv, sink, q_pos0, kv_pos0, m, W, R,
                 softmax_scale, rope_base, out_dtype, return_lse, workspace, out)


# ----------------------------------------------------------------- FP8 entry cache
def quantize_entries_fp8(ckv, R=64, codes=None, scales=None, rope=None):
    """FP8 entry cache of ckv [..., D] (BF16 or FP32): E4M3 codes of the first
    D-R dims with one power-of-two scale per entry, the last R dims in BF16
    -> (codes uint8 [..., D-R], scales uint8 [...], rope BF16 [..., R])."""
    _need_contig(ckv)
    D = ckv.shape[-1]
    rows = ckv.numel() // D if D else 0
    lead = ckv.shape[:-1]
    if codes is None:
        codes = torch.empty(lead + (D - R,), dtype=torch.uint8, device=ckv.device)
    if scales is None:
        scales = torch.empty(lead, dtype=torch.uint8, device=ckv.device)
    if rope is None:
        rope = torch.empty(lead + (R,), dtype=torch.bfloat16, device=ckv.device)
    st = _lib.lcsa_quantize_entries_fp8(_p(ckv), rows, D, R, _dt(ckv), _p(codes), _p(scales), _p(rope),
                                        _stream(ckv.device))
    _check(st, "quantize_entries_fp8")
    return codes, scales, rope


def _attn_fp8(fn, name, sparse, q, cache, idx, kv, sink, q_pos0, kv_pos0, m, W, R, softmax_scale, rope_base,
              out_dtype, return_lse, workspace, out):
    codes, scales, rope = cache
    _need_contig(q, codes, scales, rope, idx, kv, sink)
    B, Tq, H, D = q.shape
    Nc = codes.shape[1]
    dev = q.device
    if out is None:
        out = torch.empty((B, Tq, H, D), dtype=out_dtype, device=dev)
    lse = torch.empty((B, Tq, H), dtype=torch.float32, device=dev) if return_lse else None
    k = idx.shape[2] if idx is not None else 0
    a = AttnArgs(_p(q), None, _p(idx), _p(kv), _p(sink), B, Tq, H, D, R, Nc, k, kv.shape[1], int(q_pos0),
                 int(kv_pos0), m, W, float(softmax_scale), float(rope_base), _dt(q), _p(out), _dt(out), _p(lse))
    e = Fp8Entries(_p(codes), _p(scales), _p(rope))
    need = int(_lib.lcsa_attn_workspace(ctypes.byref(a), sparse))
    if need > 0 and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_n = 0 if workspace is None else workspace.numel()
    st = fn(ctypes.byref(a), ctypes.byref(e), _p(workspace), ws_n, _stream(dev))
    _check(st, name)
    return (out, lse) if return_lse else out


def csa_sparse_attn_fp8(q, cache, idx, kv, sink, q_pos0, kv_pos0, m=4, W=128, R=64, softmax_scale=0.0,
                        rope_base=10000.0, out_dtype=torch.float32, return_lse=False, workspace=None, out=None):
    """CSA core attention with the entries in the FP8 cache (codes, scales, rope)."""
    return _attn_fp8(_lib.lcsa_csa_sparse_attn_fp8, "csa_sparse_attn_fp8", 1, q, cache, idx, kv, sink, q_pos0,
                     kv_pos0, m, W, R, softmax_scale, rope_base, out_dtype, return_lse, workspace, out)


def hca_dense_attn_fp8(q, cache, kv, sink, q_pos0, kv_pos0, m=128, W=128, R=64, softmax_scale=0.0,
                       rope_base=10000.0, out_dtype=torch.float32, return_lse=False, workspace=None, out=None):
    """HCA core attention with the entries in the FP8 cache (codes, scales, rope)."""
    return _attn_fp8(_lib.lcsa_hca_dense_attn_fp8, "hca_dense_attn_fp8", 0, q, cache, None, kv, sink, q_pos0,
                     kv_pos0, m, W, R, softmax_scale, rope_base, out_dtype, return_lse, workspace, out)
