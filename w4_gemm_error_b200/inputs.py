"""Seeded synthetic inputs for the W4 + gated-EC linear layer.

This module only draws random numbers and rounds them to bf16.  It holds none
of the layer's arithmetic (no quantisation, no products with the weights), so
that both the CUDA path and the fp64 oracle can be fed from it without sharing
any code of the method.

Recipe (the pages run Llama-class models on perplexity datasets -- SPEAR,
Abstract -- which are not available here; these draws stand in for them):

* x   ~ N(0, 1) per element, with a fixed seeded set of round(frac * K) input
        channels multiplied by 20 (activation outlier channels);
* W   ~ N(0, 0.02); optionally round(frac * N) seeded output rows times 5;
* A, B ~ N(0, 0.01);
* w_g ~ N(0, 1/sqrt(K)) (standard deviation 1/sqrt(K)), b_g = 0 unless a
        target fraction of open gates is asked for (see ``gate_bias_for``).

Every draw is float64 from NumPy's PCG64, cast to float32, then rounded to
bf16 with round-to-nearest-even (torch's float32 -> bfloat16 cast).  Each
tensor has its own child seed, so the weights of a layer do not change when
only the number of tokens M changes.
"""
from __future__ import annotations

import dataclasses
from statistics import NormalDist

import numpy as np
import torch

_STREAMS = ("x", "x_outliers", "W", "W_row_outliers", "A", "B", "wg")


def _rngs(seed: int) -> dict:
    children = np.random.SeedSequence(seed).spawn(len(_STREAMS))
    return {name: np.random.Generator(np.random.PCG64(c)) for name, c in zip(_STREAMS, children)}


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float64/float32 numpy array -> torch.bfloat16 CPU tensor (RNE)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit pattern of a bf16 CPU tensor (what the oracle reads)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def outlier_channels(seed: int, K: int, frac: float) -> np.ndarray:
    """Sorted indices of the round(frac*K) input channels scaled x20."""
    n = int(round(frac * K))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rngs(seed)["x_outliers"].choice(K, size=n, replace=False)).astype(np.int64)


def gate_bias_for(wg: torch.Tensor, x_std: np.ndarray, frac_open: float) -> float:
    """Gate bias that opens about ``frac_open`` of the tokens (g > 0.5).

    The logit x.w_g of a token drawn from the recipe is normal with mean 0 and
    variance sum_k w_g[k]^2 * std(x_k)^2, so shifting it by -z*sigma with
    z = Phi^-1(1 - frac_open) leaves ``frac_open`` of the tokens above 0 in
    expectation.  Only the generating distributions are used, not the drawn x.
    """
    w = wg.float().double().numpy()
    sigma = float(np.sqrt(np.sum(w * w * x_std * x_std)))
    return float(-NormalDist().inv_cdf(1.0 - frac_open) * sigma)


@dataclasses.dataclass
class Layer:
    K: int
    N: int
    r: int
    W: torch.Tensor    # bf16 [N, K]
    A: torch.Tensor    # bf16 [K, r]
    B: torch.Tensor    # bf16 [r, N]
    wg: torch.Tensor   # bf16 [K]
    b_g: float
    outliers: np.ndarray  # input channels scaled x20


def make_layer(K: int, N: int, r: int, seed: int = 0, *, x_outlier_frac: float = 0.01,
               w_row_outlier_frac: float = 0.0, ab_std: float = 0.01, w_std: float = 0.02,
               gate_open_frac: float | None = None) -> Layer:
    g = _rngs(seed)
    W = g["W"].standard_normal((N, K)) * w_std
    n_rows = int(round(w_row_outlier_frac * N))
    if n_rows:
        rows = g["W_row_outliers"].choice(N, size=n_rows, replace=False)
        W[rows, :] *= 5.0
    A = g["A"].standard_normal((K, r)) * ab_std
    B = g["B"].standard_normal((r, N)) * ab_std
    wg = to_bf16(g["wg"].standard_normal(K) * (1.0 / np.sqrt(K)))
    outl = outlier_channels(seed, K, x_outlier_frac)
    b_g = 0.0
    if gate_open_frac is not None:
        x_std = np.ones(K)
        x_std[outl] = 20.0
        b_g = gate_bias_for(wg, x_std, gate_open_frac)
    return Layer(K, N, r, to_bf16(W), to_bf16(A), to_bf16(B), wg, b_g, outl)


def make_x(M: int, K: int, seed: int = 0, *, x_outlier_frac: float = 0.01, stream: int = 0) -> torch.Tensor:
    """Activations bf16 [M, K]; ``stream`` picks an independent batch of tokens."""
    ss = np.random.SeedSequence([seed, 7919, stream])
    x = np.random.Generator(np.random.PCG64(ss)).standard_normal((M, K))
    outl = outlier_channels(seed, K, x_outlier_frac)
    if outl.size:
        x[:, outl] *= 20.0
    return to_bf16(x)


# Workloads, named by what they are (shapes of Llama-class linears).
WORKLOADS = {
    # single small linear: a latency / parity case
    "tiny_16x256x256_r8": dict(Ms=(16,), K=256, N=256, r=8, x_outlier_frac=0.0),
    # decode, attention q/o projection of a 4096-wide model
    "decode_qo_4096x4096_r32": dict(Ms=(1, 4, 16), K=4096, N=4096, r=32),
    # decode, MLP projections of an 8B-class model (hidden 4096, intermediate 14336)
    "decode_mlp_gateup_4096x14336_r64": dict(Ms=(1, 16, 64, 128), K=4096, N=14336, r=64),
    "decode_mlp_down_14336x4096_r64": dict(Ms=(1, 16, 64, 128), K=14336, N=4096, r=64),
    # prefill, MLP gate/up projection with heavy rows and ~30% open gates
    "prefill_mlp_4096x14336_r64": dict(Ms=(2048, 4096), K=4096, N=14336, r=64,
                                       w_row_outlier_frac=0.005, gate_open_frac=0.3),
}

# Linears of a 1B-class decoder (hidden 2048, intermediate 8192, 16 layers).
STACK_1B = dict(hidden=2048, inter=8192, kv=512, layers=16, ec_layers=4, r=32,
                decode_M=64, prefill_M=1024)
STACK_1B_PROJ = (  # name, K, N
    ("q", 2048, 2048), ("k", 2048, 512), ("v", 2048, 512), ("o", 2048, 2048),
    ("gate", 2048, 8192), ("up", 2048, 8192), ("down", 8192, 2048),
)


def stack_ec_layers(seed: int = 0, layers: int = 16, count: int = 4) -> list[int]:
    """The seeded set of decoder layers whose projections carry an EC."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 104729])))
    return sorted(int(i) for i in rng.choice(layers, size=count, replace=False))
