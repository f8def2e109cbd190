"""Device-side failure detection without a GPU fault.

A testing hook (harp_test_set_faults) shortens every bounded device wait to 1 ms and
makes one wait impossible to satisfy: the dequant-GEMV's first CTA skips one stage of its
weight ring, or one grid barrier of the fused decode step gets a target one above the
grid. The wait must run out, record HARP_ERR_TIMEOUT and its site in the device status
word, end the kernel cleanly, and leave the context usable: the next normal call on the
same device must match the oracle again. No trap, assert or bad address is involved.
"""
import numpy as np
import pytest

import oracle
from harp_cases import device_layer, oracle_layer, rel_l2
from rotated_bit_matmul_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GATE = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotated_bit_matmul_b200 import build_lib, _lib
    build_lib.build()
    _lib.load()
    import rotated_bit_matmul_b200 as rb
    yield
    rb.harp_test_set_faults()
    torch.cuda.synchronize()
    rb.harp_device_status()


def _expect_timeout(sites):
    import rotated_bit_matmul_b200 as rb
    torch.cuda.synchronize()
    with pytest.raises(rb.HarpError) as e:
        rb.harp_device_status()
    assert e.value.status == 5, e.value
    site = int(str(e.value).rsplit("site", 1)[1].strip())
    assert site in sites, e.value
    rb.harp_device_status()  # cleared by the read


def test_gemv_ring_wait_runs_out_and_the_next_call_is_clean():
    import rotated_bit_matmul_b200 as rb
    case = oracle_layer(1024, 1024, 1024, 256, 2, workload=8)
    L = device_layer(case)
    x = synth.activations(1, 1024, 8, step=1)
    xd = torch.from_numpy(x).to("cuda", torch.bfloat16)
    rb.harp_test_set_faults(wait_limit_us=1000, gemv_skip_stage=0)
    try:
        L(xd, out_dtype=torch.float32)
        # site 2: a consumer's wait for the stage that never lands; 1: the producer's wait
        # for the slot the consumers never free
        _expect_timeout({1, 2})
    finally:
        rb.harp_test_set_faults()
    got = L(xd, out_dtype=torch.float32).cpu().numpy()
    rb.harp_device_status()
    L.close()
    assert rel_l2(got, oracle.linear_fwd(case["lay"], x.astype(np.float64))) < GATE


def test_fused_step_barrier_wait_runs_out_and_the_next_step_is_clean():
    import rotated_bit_matmul_b200 as rb
    dims = (4096, 1024, 32, 2, 128)
    hidden, ffn, nh, nkv, hd = dims
    shapes = [(nh * hd, hidden), (nkv * hd, hidden), (nkv * hd, hidden), (hidden, nh * hd), (ffn, hidden),
              (ffn, hidden), (hidden, ffn)]
    cases = [oracle_layer(o, i, 256 if i == ffn else i, 256 if o == ffn else o, 2, 8, 0, k)
             for k, (o, i) in enumerate(shapes)]
    layers = [device_layer(c) for c in cases]
    S = rb.HarpStack(layers, *dims)
    assert S.uses_fused_step(1)
    x = synth.activations(1, hidden, 8, step=2)
    xd = torch.from_numpy(x).to("cuda", torch.bfloat16)
    rb.harp_test_set_faults(wait_limit_us=1000, decode_barrier=0)
    try:
        S.step(xd)
        _expect_timeout(set(range(60, 70)))
    finally:
        rb.harp_test_set_faults()
    got = S.step(xd).cpu().numpy()
    rb.harp_device_status()
    want = oracle.stack_step([c["lay"] for c in cases], *dims, x.astype(np.float64))
    S.close()
    for l in layers:
        l.close()
    assert rel_l2(got, want) < GATE
