"""Workload shapes of the W4A16 decode and prefill cases.

The layer shapes follow the model families the TinyChat README benchmarks
("Speed Benchmarks": LLaMA-2-7B, LLaMA-3-8B; the 70B model it serves) and the
Falcon-180B deployment the TensorRT-LLM news item describes. Each linear layer
is y = x . W^T with W stored [N][K] (N output channels, K input channels),
group size 128 along K ("--w_bit 4 --q_group_size 128" in the README's Usage
section, step 3).
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Layer:
    name: str
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    name: str
    config_id: int
    layers: tuple
    batches: tuple
    w_std: float = 0.02
    x_std: float = 1.0
    outlier_frac: float = 0.0   # fraction of input channels scaled by outlier_mult
    outlier_mult: float = 1.0
    group: int = 128
    notes: str = field(default="", compare=False)

    def layer(self, name: str) -> Layer:
        for l in self.layers:
            if l.name == name:
                return l
        raise KeyError(name)


def outlier_count(K: int, frac: float) -> int:
    """round(frac * K) distinct input channels (half away from zero)."""
    return int(frac * K + 0.5)


WORKLOADS = {
    "single_4096": Workload(
        "single_4096", 0, (Layer("linear", 4096, 4096),), (1,),
        notes="one 4096x4096 W4A16 GEMV at M=1"),
    "llama2_7b_decode": Workload(
        "llama2_7b_decode", 1,
        (Layer("qkv", 4096, 12288), Layer("o_proj", 4096, 4096),
         Layer("gate_up", 4096, 22016), Layer("down", 11008, 4096)), (1,),
        notes="LLaMA-2-7B decoder-layer linear set at M=1"),
    "llama3_8b_decode": Workload(
        "llama3_8b_decode", 2,
        (Layer("qkv", 4096, 6144), Layer("o_proj", 4096, 4096),
         Layer("gate_up", 4096, 28672), Layer("down", 14336, 4096)), (1, 4, 8, 16, 32),
        notes="LLaMA-3-8B (GQA: 32 q heads + 2x8 kv heads, head dim 128) decode batch sweep"),
    "llama2_70b_decode": Workload(
        "llama2_70b_decode", 3,
        (Layer("qkv", 8192, 10240), Layer("o_proj", 8192, 8192),
         Layer("gate_up", 8192, 57344), Layer("down", 28672, 8192)), (1, 8, 32),
        w_std=0.01, outlier_frac=0.01, outlier_mult=20.0,
        notes="LLaMA-2-70B-shaped decode with 1% of input channels scaled x20"),
    "prefill": Workload(
        "prefill", 4,
        (Layer("llama3_gate_up", 4096, 28672), Layer("llama3_down", 14336, 4096),
         Layer("falcon180b", 14848, 59392)), (512, 2048, 8192),
        notes="prefill (context-stage) tensor-core path"),
}
