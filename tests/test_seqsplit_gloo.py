"""Sequence-parallel prefill on CPU ranks (gloo): each rank compresses its
token range (with the halo before it), one all-gather per layer exchanges the
entries (and the CSA indexer keys), and each rank's indexer, top-k and
attention over its own queries give exactly the rows of the unsharded run.
The compute steps are the oracle's; the split, halos and gather are the
package's (long_context_compressed_softmax_b200.seqsplit)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import lcsa_oracle as O
from workloads import gen
from workloads.configs import get_config


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_fns():
    def compress_entries(kv, gate, kv_pos0, m, window, j0, n):
        L = (j0 + n) * m                              # rows below kv_pos0 are never read
        fk = np.zeros((L, kv.shape[1]))
        fg = np.zeros((L, kv.shape[1]))
        hi = min(L, kv_pos0 + kv.shape[0])
        fk[kv_pos0:hi] = kv[:hi - kv_pos0].numpy()
        fg[kv_pos0:hi] = gate[:hi - kv_pos0].numpy()
        return torch.from_numpy(O.compress(fk, fg, m, window)[j0:j0 + n])

    def indexer_topk(q_idx, w, k_idx, q_pos0, m, k):
        return torch.from_numpy(O.indexer_topk(q_idx.numpy(), w.numpy(), k_idx.numpy(), q_pos0, m, k)[0])

    def csa_attn(q, ckv, idx, kv, sink, q_pos0, kv_pos0, m, W, R):
        o, _ = O.csa_sparse_attn(q.numpy()[None], ckv.numpy()[None], idx.numpy()[None], kv.numpy()[None], q_pos0,
                                 kv_pos0, m, W, sink.numpy(), R)
        return torch.from_numpy(o)

    def hca_attn(q, ckv, kv, sink, q_pos0, kv_pos0, m, W, R):
        o, _ = O.hca_dense_attn(q.numpy()[None], ckv.numpy()[None], kv.numpy()[None], q_pos0, kv_pos0, m, W,
                                sink.numpy(), R)
        return torch.from_numpy(o)

    return {"compress_entries": compress_entries, "indexer_topk": indexer_topk, "csa_attn": csa_attn,
            "hca_attn": hca_attn}


def _inputs(cfg):
    x = gen.make_layer_inputs(cfg, device="cpu", unit_scale=True)
    return {k: v[0].double() if k != "sink" else v.double() for k, v in x.items()}


def _unsharded(cfg, x, kind):
    """The oracle chain on the whole sequence."""
    kv, gate = x["kv"].numpy(), x["gate"].numpy()
    sink = x["sink"].numpy()
    if kind == "csa":
        ckv = O.csa_compress(kv, gate, cfg.m)
        idx, _ = O.indexer_topk(x["q_idx"].numpy(), x["w"].numpy(), x["k_idx"].numpy(), 0, cfg.m, cfg.k)
        o, _ = O.csa_sparse_attn(x["q"].numpy()[None], ckv[None], idx[None], kv[None], 0, 0, cfg.m, cfg.W, sink,
                                 cfg.R)
    else:
        ckv = O.hca_compress(kv, gate, cfg.m_hca)
        o, _ = O.hca_dense_attn(x["q"].numpy()[None], ckv[None], kv[None], 0, 0, cfg.m_hca, cfg.W, sink, cfg.R)
    return o


def _worker(rank, world, port, out):
    from long_context_compressed_softmax_b200 import seqsplit as S
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = get_config("tiny")
        x = _inputs(cfg)
        ranges = S.plan_ranges(cfg.T, world, cfg.m, cfg.m_hca, cfg.W)
        rr = ranges[rank]
        res = {}
        for kind in ("csa", "hca"):
            m = cfg.m if kind == "csa" else cfg.m_hca
            j0, j1 = S.local_entries(rr, m)
            xl = {"kv": x["kv"][rr.kv_pos0:rr.t1], "gate": x["gate"][rr.kv_pos0:rr.t1],
                  "q": x["q"][rr.t0:rr.t1], "sink": x["sink"]}
            if kind == "csa":
                xl.update(q_idx=x["q_idx"][rr.t0:rr.t1], w=x["w"][rr.t0:rr.t1], k_idx=x["k_idx"][j0:j1])
            got = S.prefill_layer(kind, xl, rr, ranges, cfg, _oracle_fns())
            ref = _unsharded(cfg, x, kind)[rr.t0:rr.t1]
            res[kind] = float(np.abs(got.numpy() - ref).max())
        out[rank] = (rr.t0, rr.t1, rr.kv_pos0, res)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sequence_split_equals_unsharded(world):
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    # the ranges tile [0, T) on HCA-block boundaries
    cover = sorted((t0, t1) for t0, t1, _, _ in res.values())
    assert cover[0][0] == 0 and cover[-1][1] == 1024
    assert all(a[1] == b[0] and a[0] % 128 == 0 for a, b in zip(cover, cover[1:]))
    for rank, (t0, t1, kv_pos0, errs) in res.items():
        assert kv_pos0 == max(0, t0 - 63)                   # halo: max(m, W-1) rows
        for kind, e in errs.items():
            assert e <= 1e-12, (rank, kind, e)


def test_plan_ranges_rules():
    from long_context_compressed_softmax_b200 import seqsplit as S
    r = S.plan_ranges(131072, 8, 4, 128, 128)
    assert [x.t1 - x.t0 for x in r] == [16384] * 8 and r[0].kv_pos0 == 0 and r[1].kv_pos0 == 16384 - 127
    r = S.plan_ranges(1280, 3, 4, 128, 4)                  # 10 blocks over 3 ranks: 3, 3, 4
    assert [(x.t0, x.t1) for x in r] == [(0, 384), (384, 768), (768, 1280)]
    assert r[1].kv_pos0 == 384 - 4                        # the CSA halo (m) exceeds W - 1
    with pytest.raises(ValueError):
        S.plan_ranges(1000, 2, 4, 128, 128)
    assert S.local_entries(r[1], 4) == (96, 192) and S.local_entries(r[1], 128) == (3, 6)
