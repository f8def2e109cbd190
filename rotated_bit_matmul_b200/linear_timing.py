"""Device time of harp_linear_fwd on synthetic rotated layers, with a cold L2.

    python -m rotated_bit_matmul_b200.linear_timing [--batches 1,16,64,256] [--bits 2]

For each Llama-2-7B linear shape (4096x4096, 11008x4096, 4096x11008) it builds enough
distinct layers that their packed weights together exceed the 126 MB L2 of a B200. It
captures one CUDA graph that calls every layer once at the given batch, replays the graph
and reports the time per call. The call covers the input butterfly, the GEMV
(batch < 16) or the operand prep and the tensor-core kernel (batch >= 16), and the output
butterfly. One JSON line is printed per (shape, batch):
    weight_gbs   packed codes + scale/zero bytes per second
    tflops       2 * n_out * n_in * batch per second
"""
from __future__ import annotations

import argparse
import json

import numpy as np

SHAPES = [(4096, 4096, 4096, 4096), (11008, 4096, 4096, 256), (4096, 11008, 256, 4096)]
L2_BYTES = 126 * 2 ** 20


def _layers(n_out, n_in, w_in, w_out, bits, count, device):
    import torch
    import rotated_bit_matmul_b200 as rb
    from rotated_bit_matmul_b200 import synth
    W = synth.device_weights(n_out, n_in, 3, 0, 0, device=device)
    thV, sV = synth.butterfly_params(n_in, w_in, 3, 0, 0, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, 3, 0, 0, "U")
    thV, thU = torch.from_numpy(thV).to(device), torch.from_numpy(thU).to(device)
    sV, sU = torch.from_numpy(sV).to(device), torch.from_numpy(sU).to(device)
    codes, sz = rb.harp_quantize_weights(rb.rotate_weights_device(W, thV, sV, w_in, thU, sU, w_out), bits, 64)
    del W
    return [rb.HarpLayer(n_in, n_out, bits, w_in, w_out, thV, sV, thU, sU, codes.clone(), sz.clone())
            for _ in range(count)]


def time_shape(n_out, n_in, w_in, w_out, bits, batches, reps=10, device="cuda", xdtype=None, min_layers=4):
    import torch
    xdtype = xdtype or torch.bfloat16
    wbytes = n_out * n_in * bits // 8 + n_out * (n_in // 64) * 4
    count = max(min_layers, int(np.ceil(1.5 * L2_BYTES / wbytes)))
    layers = _layers(n_out, n_in, w_in, w_out, bits, count, device)
    out = []
    for batch in batches:
        x = torch.randn(batch, n_in, device=device).to(xdtype)
        y = torch.empty(batch, n_out, device=device)
        ws = layers[0].workspace(batch)
        st = torch.cuda.Stream(device)
        with torch.cuda.stream(st):
            for L in layers:
                L(x, out=y, workspace=ws)
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for L in layers:
                L(x, out=y, workspace=ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        with torch.cuda.stream(st):
            for _ in range(3):
                g.replay()
            st.synchronize()
            for _ in range(reps):
                e0.record(st)
                g.replay()
                e1.record(st)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) / count)
        us = float(np.median(ts)) * 1e3
        abytes = x.element_size() * batch * n_in + 4 * batch * n_out  # activations in and out
        out.append(dict(n_out=n_out, n_in=n_in, bits=bits, batch=batch, layers=count, us_per_call=round(us, 3),
                        weight_gbs=round(wbytes / us / 1e3, 1), alg_bytes=wbytes + abytes,
                        alg_gbs=round((wbytes + abytes) / us / 1e3, 1),
                        tflops=round(2 * n_out * n_in * batch / us / 1e6, 2)))
        del g
    for L in layers:
        L.close()
    torch.cuda.empty_cache()
    return out


def _mr_plan(radices, seed, device):
    import torch
    import rotated_bit_matmul_b200 as rb
    rng = np.random.default_rng(seed)
    d = int(np.prod(radices))
    npar = sum((d // b) * (1 if b == 2 else b * (b - 1) // 2) for b in radices)
    th = torch.from_numpy(rng.uniform(-0.05, 0.05, npar).astype(np.float32)).to(device)
    sg = torch.from_numpy((rng.integers(0, 2, d) * 2 - 1).astype(np.int8)).to(device)
    ga = torch.from_numpy(np.concatenate([rng.standard_normal(b * b) for b in radices]).astype(np.float32)).to(device)
    return rb.HarpMixedRadix(radices, th, sg, ga)


def time_mixed_radix(side, bits=2, batch=1, reps=10, device="cuda"):
    """The 7B FFN linears with their 11008-wide side as one mixed-radix butterfly (2^8 * 43)
    instead of 43 independent 256-wide blocks: side "U" times gate/up 11008x4096, side "V"
    down 4096x11008. Returns the time per call of both layers, on the same random codes
    (the timing does not depend on their values), each over enough copies to keep L2 cold."""
    import torch
    import rotated_bit_matmul_b200 as rb
    from rotated_bit_matmul_b200 import synth
    n_out, n_in = (11008, 4096) if side == "U" else (4096, 11008)
    radices_ffn = [2] * 8 + [43] if side == "U" else [43] + [2] * 8
    wbytes = n_out * n_in * bits // 8 + n_out * (n_in // 64) * 4
    count = max(4, int(np.ceil(1.5 * L2_BYTES / wbytes)))
    g = torch.Generator(device=device).manual_seed(5)
    codes = torch.randint(0, 256, (n_out * n_in * bits // 8,), dtype=torch.uint8, device=device, generator=g)
    sz = torch.full((n_out * (n_in // 64),), 0x3C003C00, dtype=torch.int64, device=device).to(torch.int32)
    p_ffn = _mr_plan(radices_ffn, 1, device)
    p_h = _mr_plan([2] * 12, 2, device)  # the hidden side: the same radix-2 stages as the block-diagonal one
    V, U = (p_h, p_ffn) if side == "U" else (p_ffn, p_h)
    w_in, w_out = (4096, 256) if side == "U" else (256, 4096)
    thV, sV = synth.butterfly_params(n_in, w_in, 3, 0, 0, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, 3, 0, 0, "U")
    dev = lambda a: torch.from_numpy(a).to(device)
    res = {}
    for kind in ("block_diagonal", "mixed_radix"):
        cs = [codes.clone() for _ in range(count)]
        ss = [sz.clone() for _ in range(count)]
        if kind == "mixed_radix":
            layers = [rb.HarpLayer.mixed_radix(V, U, bits, c, z) for c, z in zip(cs, ss)]
        else:
            layers = [rb.HarpLayer(n_in, n_out, bits, w_in, w_out, dev(thV), dev(sV), dev(thU), dev(sU), c, z)
                      for c, z in zip(cs, ss)]
        x = torch.randn(batch, n_in, device=device).to(torch.bfloat16)
        y = torch.empty(batch, n_out, device=device)
        ws = layers[0].workspace(batch)
        st = torch.cuda.Stream(device)
        with torch.cuda.stream(st):
            for L in layers:
                L(x, out=y, workspace=ws)
        st.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=st):
            for L in layers:
                L(x, out=y, workspace=ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        with torch.cuda.stream(st):
            for _ in range(3):
                gr.replay()
            st.synchronize()
            for _ in range(reps):
                e0.record(st)
                gr.replay()
                e1.record(st)
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) / count)
        res[kind] = round(float(np.median(ts)) * 1e3, 3)
        del gr
        for L in layers:
            L.close()
    torch.cuda.empty_cache()
    return dict(n_out=n_out, n_in=n_in, side=side, radices=radices_ffn, batch=batch, layers=count,
                us_block_diagonal=res["block_diagonal"], us_mixed_radix=res["mixed_radix"],
                alg_bytes=wbytes + 2 * batch * n_in + 4 * batch * n_out)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--batches", default="1,16,64,256")
    ap.add_argument("--bits", type=int, default=2)
    ap.add_argument("--shapes", default="0,1,2", help="indices into the 7B linear shapes")
    args = ap.parse_args()
    batches = [int(b) for b in args.batches.split(",")]
    for i in (int(s) for s in args.shapes.split(",")):
        for r in time_shape(*SHAPES[i], args.bits, batches):
            print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
