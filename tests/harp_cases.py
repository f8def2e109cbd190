"""Shared helpers for the parity tests: seeded inputs -> oracle-prepared layers ->
device copies of exactly the same parameters and packed codes."""
from __future__ import annotations

import numpy as np

import oracle
from rotated_bit_matmul_b200 import synth


def rel_l2(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def oracle_layer(n_out, n_in, w_in, w_out, bits, workload=2, layer=0, linear=0):
    """Seeded W, theta and signs, rotated/quantized/packed by the oracle."""
    W = synth.weights(n_out, n_in, workload, layer, linear)
    thV, sV = synth.butterfly_params(n_in, w_in, workload, layer, linear, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, workload, layer, linear, "U")
    lay, q, s16, z16, Wr = oracle.prepare_layer(W, bits, w_in, w_out, thV, sV, thU, sU)
    return dict(W=W, thV=thV, sV=sV, thU=thU, sU=sU, lay=lay, q=q, s16=s16, z16=z16, Wr=Wr,
                n_in=n_in, n_out=n_out, w_in=w_in, w_out=w_out, bits=bits)


def device_layer(case, device="cuda"):
    import torch
    from rotated_bit_matmul_b200 import HarpLayer
    lay = case["lay"]
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dt)
    codes = torch.from_numpy(lay.packed.copy()).to(device)
    sz = torch.from_numpy(lay.sz.reshape(-1).view(np.int32).copy()).to(device)
    return HarpLayer(case["n_in"], case["n_out"], case["bits"], case["w_in"], case["w_out"],
                     t(case["thV"], torch.float32), t(case["sV"], torch.int8),
                     t(case["thU"], torch.float32), t(case["sU"], torch.int8), codes, sz)
