"""Workload shapes of the hybrid compressed-attention layer (CSA / HCA).

Shapes follow the DeepSeek-V4 descriptions: CSA pools every m=4 tokens
(overlapping 2m window) and keeps the top-2048 entries per query; HCA pools
every m'=128 tokens and attends densely; both add a 128-token sliding window
and a per-head sink; 64 query heads of dim 512 with the last 64 dims rotary;
a Lightning Indexer of 64 heads x 128 dims.
"""
from dataclasses import dataclass, field


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    dtype: str            # "fp32" or "bf16": storage type of every float input
    B: int                # sequences
    T: int                # tokens per sequence (prefill) / context length (decode)
    H: int = 64           # query heads
    D: int = 512          # head dim == shared K=V entry dim
    R: int = 64           # rotary dims (the last R of D)
    H_I: int = 64         # indexer heads
    D_I: int = 128        # indexer dim
    m: int = 4            # CSA stride (window 2m)
    m_hca: int = 128      # HCA block (window m')
    k: int = 2048         # CSA top-k
    W: int = 128          # sliding window (raw tokens)
    seed: int = 0
    decode: bool = False  # one query per sequence at position T
    layers: tuple = ()    # for the stack: ("csa","hca",...)
    gate_scale_by_dim: bool = False   # tiny config scales gate logits by 1/sqrt(D)
    boost_frac: float = 0.0           # decode: fraction of entries with boosted indexer affinity
    extra: dict = field(default_factory=dict)

    @property
    def Nc_csa(self):
        return self.T // self.m

    @property
    def Nc_hca(self):
        return self.T // self.m_hca


CONFIGS = {
    # Parity-sized layer: FP32, everything the oracle finishes in seconds.
    "tiny": WorkloadConfig(name="tiny", dtype="fp32", B=1, T=1024, H=4, D=64, R=32,
                           H_I=2, D_I=32, m=4, m_hca=128, k=64, W=64, seed=0,
                           gate_scale_by_dim=True),
    # Small CSA layer (profiling-sized case of the prefill kernels).
    "csa_prefill_8k": WorkloadConfig(name="csa_prefill_8k", dtype="bf16", B=1, T=8192, seed=6),
    # CSA layer prefill, T=32768.
    "csa_prefill_32k": WorkloadConfig(name="csa_prefill_32k", dtype="bf16", B=1, T=32768, seed=1),
    # HCA layer prefill, T=131072 (1024 entries).
    "hca_prefill_128k": WorkloadConfig(name="hca_prefill_128k", dtype="bf16", B=1, T=131072, seed=2),
    # Profiling-sized HCA layer and decode case (a few GB on the device).
    "hca_prefill_16k": WorkloadConfig(name="hca_prefill_16k", dtype="bf16", B=1, T=16384, seed=7),
    "csa_decode_8seq": WorkloadConfig(name="csa_decode_8seq", dtype="bf16", B=8, T=1 << 20, seed=8,
                                      decode=True, boost_frac=0.01),
    # CSA decode at 1M context: 64 sequences, one query each at position 2^20.
    "csa_decode_1m": WorkloadConfig(name="csa_decode_1m", dtype="bf16", B=64, T=1 << 20, seed=3,
                                    decode=True, boost_frac=0.01),
    # The compressors alone on one layer's kv and gate of the stack (B=2,
    # T=131072, 512 MB of inputs, larger than L2): profiling-sized case of the
    # CSA and HCA compress kernels.
    "compress_128k": WorkloadConfig(name="compress_128k", dtype="bf16", B=2, T=131072, seed=11),
    # Alternating four-layer stack CSA->HCA->CSA->HCA, B=2, T=131072.
    "stack_4layer_128k": WorkloadConfig(name="stack_4layer_128k", dtype="bf16", B=2, T=131072, seed=5,
                                        layers=("csa", "hca", "csa", "hca")),
    # Layer mixes of the two model sizes (first two layers differ, the rest
    # alternate CSA / HCA): V4-Flash opens with two pure sliding-window layers,
    # V4-Pro with two HCA layers.  Six layers, B=2, T=131072.
    "stack_flash_6layer_128k": WorkloadConfig(name="stack_flash_6layer_128k", dtype="bf16", B=2, T=131072, seed=9,
                                              layers=("swa", "swa", "csa", "hca", "csa", "hca")),
    "stack_pro_6layer_128k": WorkloadConfig(name="stack_pro_6layer_128k", dtype="bf16", B=2, T=131072, seed=10,
                                            layers=("hca", "hca", "csa", "hca", "csa", "hca")),
}


def get_config(name: str) -> WorkloadConfig:
    return CONFIGS[name]
