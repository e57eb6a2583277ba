"""The five decode workloads, by shape.

Shapes follow the attention layers of the model families the AsyncTLS pages
evaluate on (Qwen3-8B GQA, a GLM-4.7-Flash-style MLA latent, and an MQA
offload trace); see "AsyncTLS: Efficient Generative LLM Inference with
Asynchronous Two-level Sparse Attention", section 4 (Experimental Results).
The pages print no block size, K_b, token budget or channel count, so those
values are this workload set's own choices.
"""

from __future__ import annotations

import dataclasses
import math


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    description: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    qk_dim: int
    v_dim: int
    v_offset: int  # >= 0: V is the K row slice [v_offset, v_offset+v_dim) (MLA latent); -1: separate V
    ctx_len: int
    block_size: int
    K_b: int
    k: int
    n_label: int
    seed: int
    kv_std: float = 1.0
    n_outlier: int = 0
    outlier_scale: float = 8.0
    planted_per_row: int = 0  # planted tokens per (batch row, KV head)
    planted_blocks: int = 0  # 0: uniform positions over the whole context
    label_from_outliers: bool = False  # label channels start with the outlier channels
    steps: int = 1
    layers: int = 1
    offload: bool = False
    n_slots: int = 0
    q_drift: float = 0.1

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_blocks(self) -> int:
        return self.ctx_len // self.block_size

    @property
    def rows(self) -> int:
        return self.batch * self.n_kv_heads

    @property
    def kv_row_dim(self) -> int:
        """Elements stored per cached token row of the K tensor."""
        return self.qk_dim

    @property
    def separate_v(self) -> bool:
        return self.v_offset < 0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.qk_dim)

    def scaled(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


C1 = WorkloadConfig(
    name="c1_gqa8_4k",
    description="single decode step, one layer, batch 1, GQA 8:1, d=128, ctx 4096, bs 32, K_b 16, k 256, R 16",
    batch=1, n_q_heads=8, n_kv_heads=1, qk_dim=128, v_dim=128, v_offset=-1,
    ctx_len=4096, block_size=32, K_b=16, k=256, n_label=16, seed=0,
    n_outlier=4, planted_per_row=256, planted_blocks=16, label_from_outliers=False,
)

C2 = WorkloadConfig(
    name="c2_qwen3_8b_32k",
    description="Qwen3-8B-shaped decode: batch 8, 32:8 heads, d=128, ctx 32768, bs 64, K_b 64, k 2048, R 16",
    batch=8, n_q_heads=32, n_kv_heads=8, qk_dim=128, v_dim=128, v_offset=-1,
    ctx_len=32768, block_size=64, K_b=64, k=2048, n_label=16, seed=1,
    n_outlier=6, planted_per_row=64, planted_blocks=20, label_from_outliers=True,
)

C3 = WorkloadConfig(
    name="c3_mla_64k",
    description="MLA-shaped decode: batch 4, 128 heads on one 576-d latent (V = latent[:512]), ctx 65536, bs 64, K_b 128, k 4096, R 32",
    batch=4, n_q_heads=128, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0,
    ctx_len=65536, block_size=64, K_b=128, k=4096, n_label=32, seed=2,
    kv_std=math.sqrt(0.5), n_outlier=0, planted_per_row=64, planted_blocks=20,
    label_from_outliers=False,
)

C4 = WorkloadConfig(
    name="c4_mqa_offload_128k",
    description="MQA offload trace: batch 1, 64:1 heads, d=128, ctx 131072, bs 64, K_b 128, k 4096, R 16, 256-slot HBM block cache, 64 steps",
    batch=1, n_q_heads=64, n_kv_heads=1, qk_dim=128, v_dim=128, v_offset=-1,
    ctx_len=131072, block_size=64, K_b=128, k=4096, n_label=16, seed=3,
    n_outlier=6, planted_per_row=64, planted_blocks=20, label_from_outliers=True,
    steps=64, offload=True, n_slots=256,
)

C5 = WorkloadConfig(
    name="c5_qwen3_8b_36layer_120k",
    description="36-layer Qwen3-8B-shaped attention-only decode: batch 16, 32:8 heads, d=128, ctx 122880, bs 64, K_b 96, k 3072, R 16",
    batch=16, n_q_heads=32, n_kv_heads=8, qk_dim=128, v_dim=128, v_offset=-1,
    ctx_len=122880, block_size=64, K_b=96, k=3072, n_label=16, seed=4,
    n_outlier=6, planted_per_row=64, planted_blocks=20, label_from_outliers=True,
    steps=16, layers=36, offload=True, n_slots=192,
)

CONFIGS = {c.name: c for c in (C1, C2, C3, C4, C5)}
BY_INDEX = [C1, C2, C3, C4, C5]


def get_config(name_or_index) -> WorkloadConfig:
    if isinstance(name_or_index, int):
        return BY_INDEX[name_or_index]
    key = str(name_or_index).lower()
    if key in ("c1", "c2", "c3", "c4", "c5"):
        return BY_INDEX[int(key[1]) - 1]
    return CONFIGS[key]
