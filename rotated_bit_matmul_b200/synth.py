"""Seeded synthetic inputs shared by the CUDA path and the oracle.

This module holds no arithmetic of the method: it only draws weights, butterfly
parameters and activations with the shapes and distributions of the Llama-family
workloads the HARP pages evaluate (Llama 2 7B / 70B linear shapes), so that both
sides of every parity test start from identical numbers.

Seeds: ``numpy.random.default_rng([workload, layer, linear, role])``.
  workload: 1 single 1024x1024 layer, 2 the seven 7B decoder-layer linears,
            3 the batch sweep, 4 the 32-layer 7B stack, 5 the 80-layer 70B stack,
            11 the calibration-objective cases, 12 the int8-angle cases.
  linear:   0 q, 1 k, 2 v, 3 o, 4 gate, 5 up, 6 down, 7 = the step input.
  role:     0 W, 1 outlier columns, 2 theta_V, 3 s_V, 4 theta_U, 5 s_U, 6 x,
            7 calibration inputs.
Weights ~ N(0, 0.02^2) with a seeded set of outlier input columns scaled by 20;
theta ~ U(-0.05, 0.05) per pair and stage (the pi/4 Hadamard angle is added by
the method, not here); signs are Rademacher; activations ~ N(0, 1), rounded to
bf16 where the workload says bf16. Calibration inputs (the samples a layer's Hessian
proxy X^T X / N is formed from) are N(0, 1) with the layer's outlier channels x10.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

ROLE_W, ROLE_OUTLIER, ROLE_THETA_V, ROLE_SIGN_V, ROLE_THETA_U, ROLE_SIGN_U, ROLE_X, ROLE_CALIB_X = range(8)
LINEAR_NAMES = ("q", "k", "v", "o", "gate", "up", "down")
INPUT_SLOT = 7


@dataclass(frozen=True)
class LinearShape:
    name: str
    n_out: int
    n_in: int
    w_in: int   # butterfly block width on the input side (power of two, divides n_in)
    w_out: int  # butterfly block width on the output side


def llama7b_linears():
    """q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008; 256-wide blocks on 11008."""
    return [LinearShape("q", 4096, 4096, 4096, 4096), LinearShape("k", 4096, 4096, 4096, 4096),
            LinearShape("v", 4096, 4096, 4096, 4096), LinearShape("o", 4096, 4096, 4096, 4096),
            LinearShape("gate", 11008, 4096, 4096, 256), LinearShape("up", 11008, 4096, 4096, 256),
            LinearShape("down", 4096, 11008, 256, 4096)]


def llama70b_linears():
    """q/o 8192x8192, k/v 1024x8192, gate/up 28672x8192, down 8192x28672; 4096-wide blocks on 28672."""
    return [LinearShape("q", 8192, 8192, 8192, 8192), LinearShape("k", 1024, 8192, 8192, 1024),
            LinearShape("v", 1024, 8192, 8192, 1024), LinearShape("o", 8192, 8192, 8192, 8192),
            LinearShape("gate", 28672, 8192, 8192, 4096), LinearShape("up", 28672, 8192, 8192, 4096),
            LinearShape("down", 8192, 28672, 4096, 8192)]


STACK_DIMS = {
    # hidden, ffn, n_heads, n_kv_heads, head_dim
    "7b": (4096, 11008, 32, 32, 128),
    "70b": (8192, 28672, 64, 8, 128),
}


def rng(workload: int, layer: int, linear: int, role: int) -> np.random.Generator:
    return np.random.default_rng([int(workload), int(layer), int(linear), int(role)])


def n_outliers(n_in: int, workload: int) -> int:
    return 8 if workload == 1 else int(round(0.001 * n_in))


def weights(n_out: int, n_in: int, workload: int, layer: int, linear: int) -> np.ndarray:
    """fp32 [n_out, n_in]: N(0, 0.02^2) with outlier input columns scaled x20."""
    W = rng(workload, layer, linear, ROLE_W).standard_normal((n_out, n_in), dtype=np.float32)
    W *= np.float32(0.02)
    cols = rng(workload, layer, linear, ROLE_OUTLIER).permutation(n_in)[: n_outliers(n_in, workload)]
    W[:, cols] *= np.float32(20.0)
    return W


def outlier_columns(n_in: int, workload: int, layer: int, linear: int) -> np.ndarray:
    return rng(workload, layer, linear, ROLE_OUTLIER).permutation(n_in)[: n_outliers(n_in, workload)]


def butterfly_params(n: int, w: int, workload: int, layer: int, linear: int, side: str):
    """(theta fp32 [log2 w, n/2], sign int8 [n]) for side 'V' (input) or 'U' (output)."""
    m = int(w).bit_length() - 1
    assert 1 << m == w and n % w == 0
    rt, rs = (ROLE_THETA_V, ROLE_SIGN_V) if side == "V" else (ROLE_THETA_U, ROLE_SIGN_U)
    theta = rng(workload, layer, linear, rt).uniform(-0.05, 0.05, size=(m, n // 2)).astype(np.float32)
    sign = (rng(workload, layer, linear, rs).integers(0, 2, size=n, dtype=np.int8) * 2 - 1).astype(np.int8)
    return theta, sign


def calibration_inputs(n_samples: int, n_in: int, workload: int, layer: int, linear: int) -> np.ndarray:
    """fp32 [n_samples, n_in] layer inputs: N(0, 1) with the outlier channels scaled x10."""
    X = rng(workload, layer, linear, ROLE_CALIB_X).standard_normal((n_samples, n_in), dtype=np.float32)
    X[:, outlier_columns(n_in, workload, layer, linear)] *= np.float32(10.0)
    return X


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Rounds fp32 values to the nearest bf16 (ties to even); returns them as fp32."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def activations(batch: int, n: int, workload: int, step: int = 0, bf16: bool = True) -> np.ndarray:
    """fp32 [batch, n] ~ N(0,1), already rounded to bf16 values when ``bf16``."""
    x = rng(workload, step, INPUT_SLOT, ROLE_X).standard_normal((batch, n), dtype=np.float32)
    return round_to_bf16(x) if bf16 else x


def device_weights(n_out: int, n_in: int, workload: int, layer: int, linear: int, device="cuda"):
    """The same distribution drawn on the device (torch generator) for stacks too large
    to draw on the host; values differ from :func:`weights`."""
    import torch
    seed = ((int(workload) * 1000 + int(layer)) * 10 + int(linear)) * 10 + ROLE_W
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    W = torch.randn((n_out, n_in), generator=g, device=device, dtype=torch.float32) * 0.02
    cols = torch.from_numpy(outlier_columns(n_in, workload, layer, linear)).to(device)
    W[:, cols] *= 20.0
    return W
