"""harp_linear_fwd_static: the linear forward for callers that cannot allocate device
memory (code inside another framework's memory pool, real-time paths where an
allocation may block or fail, hosts that only hand over pre-registered buffers).

It takes its scratch from a fixed 2 MiB array in the library instead of a caller
workspace. These tests call it through the C ABI and compare it with harp_linear_fwd
(same tolerance as the other parity tests), twice in a row with different inputs so
that leftovers of the first call in the shared array cannot pass unnoticed, and check
that an oversized request is refused. The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

from harp_cases import device_layer, oracle_layer, rel_l2
from rotated_bit_matmul_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GATE = 2e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotated_bit_matmul_b200 import build_lib, _lib
    build_lib.build()
    return _lib.load()


def _static_call(lib, layer, x, out):
    st = lib.harp_linear_fwd_static(layer.handle, x.shape[0], ctypes.c_void_p(x.data_ptr()), 1,
                                    ctypes.c_void_p(out.data_ptr()), 0,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def test_static_scratch_matches_workspace_entry_point(lib):
    case = oracle_layer(11008, 4096, 4096, 256, 2, workload=2, linear=4)
    L = device_layer(case)
    for call, batch in enumerate((3, 1)):
        x = torch.from_numpy(synth.activations(batch, 4096, 2, step=100 + call)).to("cuda", torch.bfloat16)
        want = L(x, out_dtype=torch.float32)
        got = torch.full((batch, 11008), float("nan"), device="cuda")
        assert _static_call(lib, L, x, got) == 0, lib.harp_last_error()
        torch.cuda.synchronize()
        err = rel_l2(got.cpu().numpy(), want.cpu().numpy())
        assert err < GATE, (call, err)
    L.close()


def test_static_scratch_tensor_core_path(lib):
    """16 tokens take the tcgen05 path; a 4096 x 4096 layer needs about 1.4 MiB of its
    scratch, which fits the array. Two calls in a row, each equal to harp_linear_fwd."""
    case = oracle_layer(4096, 4096, 4096, 4096, 2, workload=3)
    L = device_layer(case)
    assert L.workspace_bytes(16) <= (2 << 20)
    for call in range(2):
        x = torch.from_numpy(synth.activations(16, 4096, 3, step=200 + call)).to("cuda", torch.bfloat16)
        want = L(x, out_dtype=torch.float32)
        got = torch.full((16, 4096), float("nan"), device="cuda")
        assert _static_call(lib, L, x, got) == 0, lib.harp_last_error()
        torch.cuda.synchronize()
        err = rel_l2(got.cpu().numpy(), want.cpu().numpy())
        assert err < GATE, (call, err)
    L.close()


def test_static_scratch_takes_no_device_memory_after_the_first_call(lib):
    """After the first call (which may load the library part holding the array), further
    calls leave the device's free memory exactly as it was."""
    case = oracle_layer(1024, 2048, 2048, 1024, 2, workload=8)
    L = device_layer(case)
    x = torch.from_numpy(synth.activations(2, 2048, 8, step=5)).to("cuda", torch.bfloat16)
    y = torch.empty((2, 1024), device="cuda")
    assert _static_call(lib, L, x, y) == 0, lib.harp_last_error()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert _static_call(lib, L, x, y) == 0, lib.harp_last_error()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    L.close()


def test_static_scratch_rejects_oversize(lib):
    import rotated_bit_matmul_b200 as rb
    n_out, n_in, batch = 65536, 4096, 16   # z alone needs 16 * 65536 * 4 bytes = 4 MiB
    dev = "cuda"
    L = rb.HarpLayer(n_in, n_out, 2, 4096, 4096, torch.zeros((12, n_in // 2), device=dev),
                     torch.ones(n_in, dtype=torch.int8, device=dev), torch.zeros((12, n_out // 2), device=dev),
                     torch.ones(n_out, dtype=torch.int8, device=dev),
                     torch.zeros(n_out * n_in // 4, dtype=torch.uint8, device=dev),
                     torch.zeros(n_out * n_in // 64, dtype=torch.int32, device=dev))
    assert L.workspace_bytes(batch) > (2 << 20)
    x = torch.zeros((batch, n_in), dtype=torch.bfloat16, device=dev)
    y = torch.empty((batch, n_out), dtype=torch.float32, device=dev)
    assert _static_call(lib, L, x, y) == 4  # HARP_ERR_WORKSPACE
    assert b"2097152" in lib.harp_last_error()
    L.close()
