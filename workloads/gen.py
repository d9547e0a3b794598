"""Seeded input generators (torch RNG, any device).

Each generator draws i.i.d. normal tensors in FP32 with an explicit seed, scales
them as the workload prescribes and rounds them once to the storage dtype, so
the CUDA path and the oracle see the same bits.  Nothing here computes any part
of the compressed-attention method.

Distributions (per the workload descriptions of the DeepSeek-V4 hybrid
attention layer):
  gate logits      N(0,1)                       (tiny config: N(0,1)/sqrt(D))
  kv, q            N(0,1)/sqrt(D)               (unit_scale=True: N(0,1))
  indexer q, k     N(0,1)/sqrt(D_I)
  indexer weights  N(0,1)/sqrt(H_I)
  sink logits      N(0,1)
"""
import math

import torch

_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


_CHUNK = 1 << 24     # elements drawn per generator call (fixes the stream for any size)


def randn_into(out: torch.Tensor, g: torch.Generator, scale=1.0):
    """Fill `out` (any float dtype) with N(0,1)*scale drawn in FP32 chunk by
    chunk and rounded once to out.dtype; no full-size FP32 temporary."""
    flat = out.view(-1)
    n = flat.numel()
    for i in range(0, n, _CHUNK):
        j = min(n, i + _CHUNK)
        x = torch.randn(j - i, generator=g, device=out.device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        flat[i:j].copy_(x)
    return out


def _randn(shape, g, device, scale=1.0, dtype=torch.float32):
    return randn_into(torch.empty(shape, dtype=dtype, device=device), g, scale)


def storage_dtype(dtype: str) -> torch.dtype:
    return _DT[dtype]


def make_compress_inputs(B, T, D, dtype="bf16", seed=0, device="cpu",
                         gate_per_channel=True, gate_scale=1.0, kv_scale=None):
    """kv [B,T,D] and gate logits [B,T,D] (or [B,T] for a per-token gate)."""
    g = _gen(seed, device)
    kv_scale = 1.0 / math.sqrt(D) if kv_scale is None else kv_scale
    kv = _randn((B, T, D), g, device, kv_scale, _DT[dtype])
    gshape = (B, T, D) if gate_per_channel else (B, T)
    gate = _randn(gshape, g, device, gate_scale, _DT[dtype])
    return {"kv": kv, "gate": gate}


def make_indexer_inputs(B, Tq, Nc, H_I=64, D_I=128, dtype="bf16", seed=0, device="cpu",
                        boost_frac=0.0, boost_sigma=3.0):
    """Indexer queries q_I [B,Tq,H_I,D_I], head weights w [B,Tq,H_I] (FP32) and
    per-entry indexer keys k_I [B,Nc,D_I].

    boost_frac > 0 (decode workload, Tq == 1): per sequence a seeded fraction of
    the entries has its key shifted by boost_sigma/sqrt(D_I) along the sign
    pattern of the head-weighted query, which makes the score distribution
    heavy-tailed (the +3 sigma boosted-affinity workload).
    """
    g = _gen(seed, device)
    q = _randn((B, Tq, H_I, D_I), g, device, 1.0 / math.sqrt(D_I), _DT[dtype])
    w = _randn((B, Tq, H_I), g, device, 1.0 / math.sqrt(H_I))
    k = _randn((B, Nc, D_I), g, device, 1.0 / math.sqrt(D_I))
    if boost_frac > 0.0:
        n_boost = max(1, int(round(boost_frac * Nc)))
        qf = q.float()
        for b in range(B):
            direction = torch.sign((w[b, 0, :, None] * qf[b, 0]).sum(0))  # [D_I]
            sel = torch.randperm(Nc, generator=g, device=device)[:n_boost]
            k[b, sel] += (boost_sigma / math.sqrt(D_I)) * direction
    k = k.to(_DT[dtype])
    return {"q_idx": q, "w": w, "k_idx": k}


def make_attn_inputs(B, Tq, H, D, Nc, Tkv, dtype="bf16", seed=0, device="cpu",
                     unit_scale=False, with_sink=True):
    """Queries q [B,Tq,H,D], compressed entries ckv [B,Nc,D], raw window rows
    kv [B,Tkv,D] and per-head sink logits [H] (FP32)."""
    g = _gen(seed, device)
    s = 1.0 if unit_scale else 1.0 / math.sqrt(D)
    q = _randn((B, Tq, H, D), g, device, s, _DT[dtype])
    ckv = _randn((B, Nc, D), g, device, s, _DT[dtype])
    kv = _randn((B, Tkv, D), g, device, s, _DT[dtype])
    sink = _randn((H,), g, device) if with_sink else None
    return {"q": q, "ckv": ckv, "kv": kv, "sink": sink}


def make_scores(rows, n_cols, seed=0, device="cpu", tie_levels=0):
    """FP32 score rows for selection tests.  tie_levels > 0 quantises the
    scores onto that many levels so that exact ties are frequent; signed
    zeros of both signs are planted."""
    g = _gen(seed, device)
    s = _randn((rows, n_cols), g, device)
    if tie_levels > 0:
        s = torch.round(s * (tie_levels / 8.0)) / (tie_levels / 8.0)
        s[s == 0] = 0.0
        neg0 = torch.rand((rows, n_cols), generator=g, device=device) < 0.5
        s = torch.where((s == 0) & neg0, torch.full_like(s, -0.0), s)
    return s.contiguous()


def make_topk_idx(B, Tq, k, n_vis, seed=0, device="cpu"):
    """Random ascending index lists [B,Tq,k] int32, -1 padded: row (b,t)
    holds min(k, n_vis[t]) distinct entries drawn from [0, n_vis[t])."""
    g = _gen(seed, "cpu")
    out = torch.full((B, Tq, k), -1, dtype=torch.int32)
    for b in range(B):
        for t in range(Tq):
            nv = int(n_vis[t])
            if nv <= 0:
                continue
            if nv <= k:
                sel = torch.arange(nv)
            else:
                sel = torch.sort(torch.randperm(nv, generator=g)[:k]).values
            out[b, t, :sel.numel()] = sel.to(torch.int32)
    return out.to(device)


def make_layer_inputs(cfg, device="cpu", unit_scale=False):
    """Every input of one CSA + HCA layer of workload `cfg`, drawn from one
    generator seeded with cfg.seed in a fixed order (kv, gate, q, indexer q,
    indexer weights, indexer keys, sink):

      kv    [B,T,D]        N(0,1)/sqrt(D)      (unit_scale: N(0,1))
      gate  [B,T,D]        N(0,1), or N(0,1)/sqrt(D) when cfg.gate_scale_by_dim
      q     [B,T,H,D]      N(0,1)/sqrt(D)      (unit_scale: N(0,1))
      q_idx [B,T,H_I,D_I]  N(0,1)/sqrt(D_I)
      w     [B,T,H_I]      N(0,1)/sqrt(H_I)    (FP32)
      k_idx [B,T//m,D_I]   N(0,1)/sqrt(D_I)    (one indexer key per CSA entry)
      sink  [H]            N(0,1)              (FP32)

    Float inputs are stored in cfg.dtype."""
    g = _gen(cfg.seed, device)
    dt = _DT[cfg.dtype]
    B, T, H, D, H_I, D_I = cfg.B, cfg.T, cfg.H, cfg.D, cfg.H_I, cfg.D_I
    s = 1.0 if unit_scale else 1.0 / math.sqrt(D)
    return {
        "kv": _randn((B, T, D), g, device, s, dt),
        "gate": _randn((B, T, D), g, device, 1.0 / math.sqrt(D) if cfg.gate_scale_by_dim else 1.0, dt),
        "q": _randn((B, T, H, D), g, device, s, dt),
        "q_idx": _randn((B, T, H_I, D_I), g, device, 1.0 / math.sqrt(D_I), dt),
        "w": _randn((B, T, H_I), g, device, 1.0 / math.sqrt(H_I)),
        "k_idx": _randn((B, T // cfg.m, D_I), g, device, 1.0 / math.sqrt(D_I), dt),
        "sink": _randn((H,), g, device),
    }
