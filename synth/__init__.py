"""Seeded synthetic inputs for the NVFP4 hot path.

Shared by the tests, the benchmark and the smoke check, and by both the CUDA path and the
CPU oracle.  It holds none of the method's arithmetic: only random draws, the placement of
outliers, the FP32 -> bf16 cast of the inputs and the workload shapes.

Value recipes (the pages train on real data; these stand in for it):
  activations : N(0, 1), then exactly floor(1 % of n) distinct positions multiplied by 50
  weights     : N(0, 0.02^2)
  gradients   : N(0, (1e-3)^2), then exactly floor(0.5 % of n) distinct positions x 100
Every tensor draws from numpy's PCG64 seeded by (workload seed, tensor id).
"""
from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round FP32 values to bf16 (nearest, ties to even) and return the bit patterns as
    uint16.  Inputs are finite."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor_id)])


def _with_spikes(rng, z: np.ndarray, frac: float, mult: float) -> np.ndarray:
    n = z.size
    k = int(np.floor(frac * n))
    if k > 0:
        pos = rng.choice(n, size=k, replace=False)
        flat = z.reshape(-1)
        flat[pos] *= np.float32(mult)
    return z


def activations(shape: Tuple[int, int], seed: int, tensor_id: int = 0,
                outlier_frac: float = 0.01, outlier_mult: float = 50.0) -> np.ndarray:
    rng = _rng(seed, tensor_id)
    z = rng.standard_normal(int(np.prod(shape)), dtype=np.float32).reshape(shape)
    return f32_to_bf16_bits(_with_spikes(rng, z, outlier_frac, outlier_mult))


def weights(shape: Tuple[int, int], seed: int, tensor_id: int = 1,
            sigma: float = 0.02) -> np.ndarray:
    rng = _rng(seed, tensor_id)
    z = rng.standard_normal(int(np.prod(shape)), dtype=np.float32).reshape(shape)
    return f32_to_bf16_bits(z * np.float32(sigma))


def gradients(shape: Tuple[int, int], seed: int, tensor_id: int = 2, sigma: float = 1e-3,
              spike_frac: float = 0.005, spike_mult: float = 100.0) -> np.ndarray:
    rng = _rng(seed, tensor_id)
    z = rng.standard_normal(int(np.prod(shape)), dtype=np.float32).reshape(shape)
    z *= np.float32(sigma)
    return f32_to_bf16_bits(_with_spikes(rng, z, spike_frac, spike_mult))


# ---- workloads -------------------------------------------------------------------------

@dataclass
class Linear:
    """One linear layer y = x . W^T with T tokens, I in-features, O out-features."""
    name: str
    T: int
    I: int
    O: int

    @property
    def gemm_flops(self) -> Dict[str, int]:
        f = 2 * self.T * self.I * self.O
        return {"fprop": f, "dgrad": f, "wgrad": f}


@dataclass
class Workload:
    name: str
    seed: int
    linears: List[Linear] = field(default_factory=list)
    description: str = ""


def fprop_small() -> Workload:
    """Single fprop linear: X [256 x 512], W [512 x 512], Y = X . W^T in FP32."""
    return Workload("fprop_t256_i512_o512", 0, [Linear("fprop", 256, 512, 512)],
                    "single fprop linear, X 256x512 activations, W 512x512 weights")


def layer_4096() -> Workload:
    """One linear layer, fwd + bwd, T = I = O = 4096."""
    return Workload("linear_t4096_i4096_o4096", 1, [Linear("linear", 4096, 4096, 4096)],
                    "one linear layer fwd+bwd, tokens 4096, in = out = 4096")


def mlp_12b() -> Workload:
    """12B-class MLP: tokens 8192, d_model 5120, up 5120 -> 20480, down 20480 -> 5120."""
    return Workload("mlp12b_t8192_d5120_ff20480", 2,
                    [Linear("up", 8192, 5120, 20480), Linear("down", 8192, 20480, 5120)],
                    "12B-class MLP, tokens 8192, up 5120->20480 and down 20480->5120, "
                    "fprop+dgrad+wgrad of each linear")


def dense_8b_layer() -> Workload:
    """8B-class dense transformer layer linears at tokens 16384, d = 4096."""
    T = 16384
    return Workload("dense8b_t16384_d4096", 4,
                    [Linear("qkv", T, 4096, 6144), Linear("o", T, 4096, 4096),
                     Linear("gate", T, 4096, 14336), Linear("up", T, 4096, 14336),
                     Linear("down", T, 14336, 4096)],
                    "8B-class dense layer linears, 4 NVFP4 layers + 1 bf16 layer")


QUANT_SWEEP_SEED = 3
QUANT_SWEEP_ROW = 4096
QUANT_SWEEP_LOG2 = list(range(20, 31))


def quant_sweep_shape(log2n: int) -> Tuple[int, int]:
    """Quantizer bandwidth sweep tensor of 2^log2n bf16 elements in rows of 4096."""
    n = 1 << log2n
    return (n // QUANT_SWEEP_ROW, QUANT_SWEEP_ROW)


def linear_inputs(lin: Linear, seed: int, layer_index: int = 0):
    """X [T x I] activations, W [O x I] weights, dY [T x O] gradients (bf16 bits)."""
    base = 16 * layer_index
    X = activations((lin.T, lin.I), seed, tensor_id=base + 0)
    W = weights((lin.O, lin.I), seed, tensor_id=base + 1)
    dY = gradients((lin.T, lin.O), seed, tensor_id=base + 2)
    return X, W, dY
