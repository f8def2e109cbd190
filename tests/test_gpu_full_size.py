"""Oracle parity of the benchmark's own configuration at full size.

The bench runs a 32-block Llama-2-7B-shaped stack of rotated 2-bit linears (weights drawn
on the device, rotated and quantized by the library) through the fused single-kernel
decode step at batch 1. These tests compare exactly that stack, in that launch
configuration, with the fp64 oracle:

* teacher-forced blocks: the input of block l is the fused step's output of the first l
  blocks (the kernel is deterministic, so it is bit for bit what the full stack feeds
  block l); the oracle runs block l alone on it, from the device's own codes and scales
  and the seeded angles and signs, and the fused step of the first l + 1 blocks must
  match it. Blocks 0, 15 and 31 (first, middle, last; grid-barrier counters up to the
  last block's);
* one whole 32-block step against the oracle's 32-block step (about 3 minutes of fp64
  work on the host cores).

Gates: rel-L2 2e-3 (the library's contract for the fp32-accumulate path) over the whole
output, and 1e-2 on the worst 256-element slice of it.
"""
import numpy as np
import pytest

import oracle
from harp_cases import rel_l2
from rotated_bit_matmul_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GATE = 2e-3
SLICE_GATE = 1e-2


@pytest.fixture(scope="module")
def bench_stack():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bench
    from rotated_bit_matmul_b200 import build_lib, _lib
    build_lib.build()
    _lib.load()
    oracle.set_threads(max(1, len(__import__("os").sched_getaffinity(0))))
    dev = torch.device("cuda", 0)
    S = bench.build_stack(bench.N_LAYERS, dev)
    assert S.uses_fused_step(1)
    yield bench, S
    S.close()
    import rotated_bit_matmul_b200 as rb
    torch.cuda.synchronize()
    rb.harp_device_status()


def _oracle_blocks(bench, S, blocks):
    """Oracle layers of the given blocks, from the device's packed codes and scale/zero and
    the seeded angles and signs the bench built them with."""
    lays = []
    for l in blocks:
        for i, s in enumerate(bench.shapes()):
            L = S.layers[7 * l + i]
            thV, sV = synth.butterfly_params(s.n_in, s.w_in, bench.WORKLOAD, l, i, "V")
            thU, sU = synth.butterfly_params(s.n_out, s.w_out, bench.WORKLOAD, l, i, "U")
            packed = L.codes.cpu().numpy()
            sz = L.scale_zero.cpu().numpy().view(np.uint16).reshape(s.n_out, s.n_in // 64, 2)
            lays.append(oracle.Layer(s.n_in, s.n_out, bench.BITS, s.w_in, s.w_out, thV, sV, thU, sU, packed, sz))
    return lays


def _fused_prefix(bench, S, n_blocks, x):
    """Output of the fused step over the first n_blocks blocks of the bench stack (fp32)."""
    import rotated_bit_matmul_b200 as rb
    if n_blocks == 0:
        return x.float()
    sub = rb.HarpStack(S.layers[:7 * n_blocks], bench.HIDDEN, bench.FFN, bench.NH, bench.NKV, bench.HD)
    assert sub.uses_fused_step(1)
    y = sub.step(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    sub.close()
    return y


def _gates(got, want, what):
    err = rel_l2(got, want)
    sl = max(rel_l2(got[..., t:t + 256], want[..., t:t + 256]) for t in range(0, want.shape[-1], 256))
    print(f"{what}: rel-L2 {err:.3e}, worst 256-slice {sl:.3e}")
    assert err < GATE, (what, err)
    assert sl < SLICE_GATE, (what, sl)


@pytest.mark.parametrize("block", [0, 15, 31])
def test_bench_stack_teacher_forced_block(bench_stack, block):
    bench, S = bench_stack
    x = torch.from_numpy(synth.activations(1, bench.HIDDEN, bench.WORKLOAD, step=21)).to("cuda", torch.bfloat16)
    x_in = _fused_prefix(bench, S, block, x)
    y = _fused_prefix(bench, S, block + 1, x)
    want = oracle.stack_step(_oracle_blocks(bench, S, [block]), bench.HIDDEN, bench.FFN, bench.NH, bench.NKV,
                             bench.HD, x_in.cpu().numpy().astype(np.float64))
    _gates(y.cpu().numpy(), want, f"block {block} of {bench.N_LAYERS}")


@pytest.mark.slow
def test_bench_stack_whole_step(bench_stack):
    """The full 32-block fused step against the oracle's 32-block step on the same input."""
    bench, S = bench_stack
    x = synth.activations(1, bench.HIDDEN, bench.WORKLOAD, step=22)
    y = S.step(torch.from_numpy(x).to("cuda", torch.bfloat16), out_dtype=torch.float32).cpu().numpy()
    want = oracle.stack_step(_oracle_blocks(bench, S, range(bench.N_LAYERS)), bench.HIDDEN, bench.FFN, bench.NH,
                             bench.NKV, bench.HD, x.astype(np.float64))
    _gates(y, want, "whole 32-block step")
