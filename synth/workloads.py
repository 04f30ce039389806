"""The five synthetic workloads of the W4A16 linear layer (shapes, seeds, tags).

Shapes are (K, N) = (input features, output features); weights are stored
[N, K].  Every tensor is drawn by ``synth`` from (seed, tag):
  * single GEMV      : M = 1, (4096, 4096), W and X seed 0
  * decode set 5120  : M = 1, hidden-5120 layer shapes, W and X seeds 1..4 in list order
  * small batch 8192 : M in {2, 4, 8, 16, 32}, hidden-8192 shapes, W seed 100 + shape index, X seed 200 + M
  * prefill 8192     : M in {512, 2048, 4096}, same weights as above, X seed 300 + M
  * decode stack     : 80 layers x hidden-8192 shapes, M = 1, W seed = layer index with
                       tag TAG_W_STACK + shape index, X (the first hidden state) seed 5000;
                       each layer's qkv / o / gate+up read the hidden state h, down reads the
                       first 28672 outputs of gate+up renormalised, and the next h is the
                       renormalised output of down
"""
from __future__ import annotations

from dataclasses import dataclass

from . import TAG_W, TAG_W_STACK

HIDDEN_5120 = [("qkv", 5120, 7680), ("o_proj", 5120, 5120), ("gate_up", 5120, 51200), ("down", 25600, 5120)]
HIDDEN_8192 = [("qkv", 8192, 10240), ("o_proj", 8192, 8192), ("gate_up", 8192, 57344), ("down", 28672, 8192)]
SMALL_BATCH_M = [2, 4, 8, 16, 32]
PREFILL_M = [512, 2048, 4096]
STACK_LAYERS = 80
STACK_X_SEED = 5000


@dataclass(frozen=True)
class Case:
    workload: str
    name: str
    M: int
    K: int
    N: int
    w_seed: int
    w_tag: int
    x_seed: int

    @property
    def code_bytes(self) -> int:
        return self.N * self.K // 2

    @property
    def meta_bytes(self) -> int:
        return self.N * (self.K // 128) * 6

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


def single_gemv() -> list[Case]:
    return [Case("single_gemv_4096", "gemv", 1, 4096, 4096, 0, TAG_W, 0)]


def decode_5120() -> list[Case]:
    return [Case("decode_hidden5120_m1", name, 1, K, N, i + 1, TAG_W, i + 1)
            for i, (name, K, N) in enumerate(HIDDEN_5120)]


def small_batch_8192(ms=SMALL_BATCH_M) -> list[Case]:
    return [Case("small_batch_hidden8192", f"{name}_m{M}", M, K, N, 100 + i, TAG_W, 200 + M)
            for M in ms for i, (name, K, N) in enumerate(HIDDEN_8192)]


def prefill_8192(ms=PREFILL_M) -> list[Case]:
    return [Case("prefill_hidden8192", f"{name}_m{M}", M, K, N, 100 + i, TAG_W, 300 + M)
            for M in ms for i, (name, K, N) in enumerate(HIDDEN_8192)]


def stack_layer(layer: int) -> list[Case]:
    return [Case("decode_stack_80x8192", f"L{layer}_{name}", 1, K, N, layer, TAG_W_STACK + i, STACK_X_SEED)
            for i, (name, K, N) in enumerate(HIDDEN_8192)]
