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
