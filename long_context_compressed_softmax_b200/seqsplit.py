"""Sequence-parallel prefill of one CSA or HCA layer across ranks (one rank per
GPU, torch.distributed for the exchange).

The queries of a sequence are split into contiguous token ranges, one per
rank, with boundaries on multiples of the HCA block m' (hence of the CSA
stride m too).  A rank

  1. compresses the entries whose own block lies in its range: CSA entry j
     pools tokens [(j-1)m, (j+1)m), so the range's first entry needs the m
     tokens before the range (a halo from the previous rank's tokens); HCA
     blocks lie inside the range;
  2. exchanges entries in ONE all-gather per layer: the compressed entries
     and, for CSA, the indexer keys of those entries (one key per entry),
     packed into one buffer;
  3. runs the indexer + top-k and the core attention for its own queries
     against the gathered entries; the sliding window reads raw rows back to
     W-1 tokens before the range (the same halo rows the rank holds).

Everything the rank needs besides the gathered entries is local, so the
all-gather is the only collective.  This is the sequence split of the
compressed-attention layer; a batch of independent sequences needs no
collective at all (each rank takes whole sequences).

The compute steps are passed in as callables, so the same plan runs the
library's kernels on GPUs (NCCL) or any other implementation of the steps
(gloo on CPU in the tests).  No TMA multicast or peer-memory load is used:
the gathered entries land in each rank's own memory.
"""
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankRange:
    """Token range [t0, t1) of one rank and the raw rows it holds,
    [kv_pos0, t1): the range plus a halo for the CSA window and the
    sliding window."""
    rank: int
    t0: int
    t1: int
    kv_pos0: int

    @property
    def rows(self):
        return self.t1 - self.kv_pos0


def plan_ranges(T, world, m, m_hca, W):
    """Contiguous query ranges of a T-token sequence, one per rank, with
    boundaries on multiples of m_hca (which must be a multiple of m), as
    equal as that allows; each with the halo rows below it:
    max(m, W - 1) rows before t0 (clipped at 0)."""
    if m_hca % m != 0:
        raise ValueError("the HCA block must be a multiple of the CSA stride")
    if T % m_hca != 0:
        raise ValueError("sequence length must be a multiple of the HCA block")
    blocks = T // m_hca
    halo = max(m, W - 1)
    out = []
    for r in range(world):
        b0 = blocks * r // world
        b1 = blocks * (r + 1) // world
        t0, t1 = b0 * m_hca, b1 * m_hca
        out.append(RankRange(r, t0, t1, max(0, t0 - halo)))
    return out


def local_entries(rr, m):
    """Entries [j0, j1) whose own block [j m, (j+1) m) lies in the rank's range."""
    return rr.t0 // m, rr.t1 // m


def all_gather_rows(x, counts, group=None):
    """Concatenate every rank's rows x [n_r, ...] in rank order (n_r =
    counts[r]); one all-gather of equally sized (padded) buffers."""
    world = len(counts)
    if world == 1:
        return x
    cap = max(counts)
    pad = x.new_zeros((cap,) + tuple(x.shape[1:]))
    pad[:x.shape[0]] = x
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad.contiguous(), group=group)
    return torch.cat([bufs[r][:counts[r]] for r in range(world)], dim=0)


def prefill_layer(kind, x, rr, ranges, cfg, fns, group=None):
    """One layer's prefill on this rank.

    kind    "csa" or "hca"
    x       this rank's inputs: kv, gate [rows, D] (raw rows kv_pos0 .. t1-1),
            q [t1-t0, H, D], sink [H]; for CSA also q_idx [t1-t0, H_I, D_I],
            w [t1-t0, H_I] and k_idx [j1-j0, D_I] (the keys of its own entries)
    rr      this rank's RankRange; ranges: every rank's
    cfg     m, m_hca, W, R, k (a WorkloadConfig or anything with those names)
    fns     compute steps (one sequence):
              compress_entries(kv, gate, kv_pos0, m, window, j0, n) -> [n, D]
              indexer_topk(q_idx, w, k_idx_all, q_pos0, m, k) -> idx [Tq, k]
              csa_attn(q, ckv_all, idx, kv, sink, q_pos0, kv_pos0, m, W, R) -> [Tq, H, D]
              hca_attn(q, ckv_all, kv, sink, q_pos0, kv_pos0, m, W, R) -> [Tq, H, D]
    Returns the attention output of the rank's queries [t1-t0, H, D].
    """
    m = cfg.m if kind == "csa" else cfg.m_hca
    window = 2 * m if kind == "csa" else m
    j0, j1 = local_entries(rr, m)
    own = fns["compress_entries"](x["kv"], x["gate"], rr.kv_pos0, m, window, j0, j1 - j0)
    counts = [local_entries(r, m)[1] - local_entries(r, m)[0] for r in ranges]
    if kind == "csa":
        # entries and indexer keys travel in one buffer: [n, D + D_I] in the entries' dtype
        D = own.shape[1]
        packed = torch.cat([own, x["k_idx"].to(own.dtype)], dim=1)
        allp = all_gather_rows(packed, counts, group)
        ckv_all = allp[:, :D].contiguous()
        k_idx_all = allp[:, D:].to(x["k_idx"].dtype).contiguous()
        idx = fns["indexer_topk"](x["q_idx"], x["w"], k_idx_all, rr.t0, m, cfg.k)
        return fns["csa_attn"](x["q"], ckv_all, idx, x["kv"], x["sink"], rr.t0, rr.kv_pos0, m, cfg.W, cfg.R)
    ckv_all = all_gather_rows(own, counts, group)
    return fns["hca_attn"](x["q"], ckv_all, x["kv"], x["sink"], rr.t0, rr.kv_pos0, m, cfg.W, cfg.R)


def library_fns(lcsa):
    """The compute steps on the library's kernels (one sequence, device tensors)."""
    def compress_entries(kv, gate, kv_pos0, m, window, j0, n):
        D = kv.shape[-1]
        cache = torch.empty((1, j0 + n, D), dtype=kv.dtype, device=kv.device)
        lcsa.compress_entries(kv[None], gate[None], kv_pos0, m, window, j0, n, cache)
        return cache[0, j0:j0 + n]

    def indexer_topk(q_idx, w, k_idx, q_pos0, m, k):
        return lcsa.indexer_topk(q_idx[None], w[None], k_idx[None], q_pos0, m, k)[0]

    def csa_attn(q, ckv, idx, kv, sink, q_pos0, kv_pos0, m, W, R):
        return lcsa.csa_sparse_attn(q[None], ckv[None], idx[None], kv[None], sink, q_pos0, kv_pos0, m, W, R)[0]

    def hca_attn(q, ckv, kv, sink, q_pos0, kv_pos0, m, W, R):
        return lcsa.hca_dense_attn(q[None], ckv[None], kv[None], sink, q_pos0, kv_pos0, m, W, R)[0]

    return {"compress_entries": compress_entries, "indexer_topk": indexer_topk, "csa_attn": csa_attn,
            "hca_attn": hca_attn}
