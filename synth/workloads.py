"""The five synthetic workloads: shapes, value distributions and seeds.

Each linear layer is described by a :class:`Layer`; its weights and its
activations come from :mod:`synth` (host, numpy) or ``synth_dev.cu``
(device) with identical float32 bits.  Seeds follow one rule,
``0x5EED0000 + 1000*config + 10*layer + matrix_id``, with separate streams for
W, the heavy-tail selection, x, the calibration tokens and the outlier
channel choice.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

import synth

CAL_TOKENS = 64


@dataclass(frozen=True)
class Layer:
    name: str
    config: int
    layer: int
    matrix_id: int
    K: int                     # input channels
    N: int                     # output rows
    M: int = 1                 # tokens
    w_kind: str = "laplace"    # "laplace" | "gauss_heavy"
    w_scale: float = 0.02      # Laplace b, or Gaussian sigma
    heavy_frac: float = 0.0
    heavy_mul: float = 1.0
    n_out: int = 4             # outlier channels
    out_factor: float = 50.0   # multiplier of the outlier channels in x
    trunk_percent: int = -1    # <0: full trunk; else per-row percentile
    group: int = 128
    residual_percent: int = 0  # 0: dense residual; > 0: that per-row percentile of |r| dropped; < 0: asymmetric groups

    @property
    def seed(self) -> int:
        return 0x5EED0000 + 1000 * self.config + 10 * self.layer + self.matrix_id

    # ---- host generation (numpy) -------------------------------------------
    def weights(self, rows=None) -> np.ndarray:
        if self.w_kind == "laplace":
            return synth.laplace_matrix(self.seed, self.N, self.K, self.w_scale, rows)
        return synth.gauss_heavy_matrix(self.seed, self.N, self.K, self.w_scale,
                                        self.heavy_frac, self.heavy_mul, rows)

    def planted_channels(self) -> np.ndarray:
        return synth.outlier_channels(self.seed, self.K, self.n_out)

    def factors(self) -> np.ndarray:
        return synth.channel_factors(self.K, self.planted_channels(), self.out_factor)

    def activations(self, M: int | None = None, rows=None) -> np.ndarray:
        return synth.activation_matrix(self.seed, synth.STREAM_X, M or self.M, self.K,
                                       self.factors(), rows)

    def calibration(self, T: int = CAL_TOKENS) -> np.ndarray:
        return synth.activation_matrix(self.seed, synth.STREAM_XCAL, T, self.K, self.factors())

    def with_(self, **kw) -> "Layer":
        d = dict(self.__dict__)
        d.update(kw)
        return Layer(**d)

    @property
    def packed_bytes(self) -> int:
        """Algorithmic bytes of the packed weights: sign (+mask) bits, INT8
        codes, fp32 group scales and fp32 row scale, per row."""
        ng = (self.K + self.group - 1) // self.group
        planes = 2 if self.trunk_percent >= 0 else 1
        per_row = planes * self.K / 8 + self.K + 4 * ng + 4
        return int(round(self.N * per_row))

    def act_bytes(self, M: int | None = None) -> int:
        """Per call of the linear: INT8 codes, token scale, outlier values and
        indices in; fp32 y out."""
        M = M or self.M
        return M * (self.K + 4 + 4 * self.n_out + 4 * self.N) + 4 * self.n_out


def n_outliers(K: int, frac: float) -> int:
    return max(1, int(np.floor(frac * K + 0.5)))


def config1() -> Layer:
    """Single 512x512 layer, batch 1, Laplace(0, 0.02) weights, 4 channels x50."""
    return Layer("single_512", 1, 0, 0, K=512, N=512, n_out=4, out_factor=50.0)


STACK_SHAPES = (("qkv", 4096, 12288), ("o", 4096, 4096), ("gate_up", 4096, 22016),
                ("down", 11008, 4096))
STACK_LAYERS = 32


def config2_layer(layer: int, mid: int) -> Layer:
    name, K, N = STACK_SHAPES[mid]
    return Layer(f"l{layer}.{name}", 2, layer, mid, K=K, N=N, n_out=n_outliers(K, 0.005),
                 out_factor=30.0)


def config2(layers: int = STACK_LAYERS) -> list[Layer]:
    """Llama-2-7B-shaped decode stack: 32 x {qkv, o, gate_up, down}, batch 1."""
    return [config2_layer(l, m) for l in range(layers) for m in range(4)]


def config3(M: int = 1) -> list[Layer]:
    """70B-shaped MLP pair, Gaussian sigma 0.015 with 0.1% entries x10,
    x with 0.25% channels x40, batch M in {1, 2, 4, 8, 16}."""
    out = []
    for mid, (K, N) in enumerate(((8192, 28672), (28672, 8192))):
        out.append(Layer(f"mlp70b_{K}x{N}_m{M}", 3, 0, mid, K=K, N=N, M=M,
                         w_kind="gauss_heavy", w_scale=0.015, heavy_frac=0.001,
                         heavy_mul=10.0, n_out=n_outliers(K, 0.0025), out_factor=40.0))
    return out


def config4() -> Layer:
    """Threshold trunk: 4096 -> 14336, per-row 60th percentile, batch 1."""
    return Layer("thresh_4096x14336", 4, 0, 0, K=4096, N=14336, n_out=n_outliers(4096, 0.005),
                 out_factor=30.0, trunk_percent=60)


def config5() -> Layer:
    """Prefill-shaped: M=2048 tokens, 4096 -> 14336."""
    return Layer("prefill_2048x4096x14336", 5, 0, 0, K=4096, N=14336, M=2048,
                 n_out=n_outliers(4096, 0.005), out_factor=30.0)
