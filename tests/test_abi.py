"""CPU checks of the C ABI: the library loads, exports every entry point include/harp.h
declares, and rejects bad arguments with a status (validation runs before any CUDA
call, so none of these touch a GPU)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "harp.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(harp_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from rotated_bit_matmul_b200 import build_lib, _lib
    build_lib.build()
    return _lib.load()


def test_library_exports_every_declared_symbol(lib):
    names = _declared()
    assert "harp_linear_fwd" in names and "harp_create_layer" in names
    for n in names:
        assert hasattr(lib, n), n


def test_binding_signatures_cover_header():
    from rotated_bit_matmul_b200 import _lib
    assert sorted(_lib.SIGNATURES) == _declared()


FAKE = ctypes.c_void_p(1 << 20)       # aligned, never dereferenced: validation fails first
MIS = ctypes.c_void_p((1 << 20) + 4)  # misaligned


@pytest.mark.parametrize("n,w,batch,x,err", [
    (1024, 3, 1, FAKE, 1),       # w not a power of two
    (1024, 16384, 1, FAKE, 1),   # w too wide
    (1000, 16, 1, FAKE, 1),      # w does not divide n
    (1024, 1024, -1, FAKE, 1),   # negative batch
    (1024, 1024, 1, MIS, 1),     # misaligned pointer
    (1024, 1024, 1, None, 1),    # null pointer
])
def test_butterfly_rejects_bad_arguments(lib, n, w, batch, x, err):
    st = lib.harp_butterfly_fwd(n, w, batch, FAKE, FAKE, x, 0, FAKE, 0, None)
    assert st == err
    assert lib.harp_last_error()


def test_butterfly_inplace_dtype_mismatch(lib):
    assert lib.harp_butterfly_inv(1024, 1024, 1, FAKE, FAKE, FAKE, 0, FAKE, 1, None) == 1


@pytest.mark.parametrize("args,err", [
    ((4096, 4096, 5, 64), 1),    # bits out of range
    ((4096, 4096, 2, 32), 2),    # unsupported group
    ((4096, 100, 2, 64), 1),     # n_in not a multiple of 64
])
def test_quantize_rejects_bad_arguments(lib, args, err):
    assert lib.harp_quantize_weights(*args, FAKE, FAKE, FAKE, None) == err


@pytest.mark.parametrize("n_in,n_out,bits,w_in,w_out,err", [
    (4096, 4096, 1, 4096, 4096, 1),    # bits
    (4000, 4096, 2, 4096, 4096, 1),    # n_in not a multiple of 256
    (4096, 4096, 2, 32, 4096, 1),      # w_in below 64
    (4096, 4096, 2, 4096, 3000, 1),    # w_out not a power of two
    (11008, 4096, 2, 4096, 4096, 1),   # w_in does not divide n_in
    (4096, 4096, 2, 16384, 4096, 1),   # w_in too wide
])
def test_create_layer_rejects_bad_arguments(lib, n_in, n_out, bits, w_in, w_out, err):
    h = ctypes.c_void_p()
    st = lib.harp_create_layer(ctypes.byref(h), n_in, n_out, bits, 64, w_in, w_out, FAKE, FAKE, FAKE, FAKE, FAKE,
                               FAKE, None)
    assert st == err and not h.value


def test_null_handles(lib):
    n = ctypes.c_size_t()
    assert lib.harp_linear_workspace_size(None, 1, ctypes.byref(n)) == 1
    assert lib.harp_linear_fwd(None, 1, FAKE, 0, FAKE, 0, FAKE, 1 << 20, None) == 1
    assert lib.harp_destroy_layer(None) == 0
    assert lib.harp_stack_destroy(None) == 0
    assert lib.harp_stack_step(None, 1, FAKE, 0, FAKE, 0, FAKE, 1 << 20, None) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    from rotated_bit_matmul_b200 import _lib
    with pytest.raises(ImportError):
        saved = _lib._lib
        _lib._lib = None
        try:
            _lib.load(str(tmp_path / "missing.so"))
        finally:
            _lib._lib = saved


def _no_gpu():
    import torch
    if torch.cuda.is_available():
        # on a GPU the calls below would reach the device with placeholder pointers
        pytest.skip("needs a machine without a CUDA device")


def test_null_theta_passes_validation(lib):
    """A null theta selects the fixed randomized Hadamard transform (Theta = 0): argument
    checks accept it, and without a GPU the calls fail only at the first CUDA call
    (HARP_ERR_CUDA), not as HARP_ERR_INVALID_ARG."""
    _no_gpu()
    h = ctypes.c_void_p()
    st = lib.harp_create_layer(ctypes.byref(h), 4096, 4096, 2, 64, 4096, 4096, None, FAKE, None, FAKE, FAKE,
                               FAKE, None)
    assert st == 3 and not h.value, lib.harp_last_error()
    assert lib.harp_butterfly_fwd(4096, 4096, 1, None, FAKE, FAKE, 0, FAKE, 0, None) == 3
    # a null sign vector is still an error
    assert lib.harp_butterfly_fwd(4096, 4096, 1, None, None, FAKE, 0, FAKE, 0, None) == 1


def test_empty_batch_is_a_no_op(lib):
    """batch 0 is valid for the butterflies and returns before any launch."""
    assert lib.harp_butterfly_fwd(4096, 4096, 0, FAKE, FAKE, FAKE, 0, FAKE, 0, None) == 0
    assert lib.harp_butterfly_inv(4096, 4096, 0, None, FAKE, FAKE, 0, FAKE, 0, None) == 0


def test_calib_workspace_size(lib):
    """Without a Hessian proxy or gradient: two fp32 copies of W, the packed codes, the
    scale/zero words and per-column fp32/fp64 vectors; each extra adds its buffers."""
    n = ctypes.c_size_t()
    assert lib.harp_calib_workspace_size(4096, 4096, 2, 4096, 4096, 0, 0, ctypes.byref(n)) == 0
    base = n.value
    nw = 4096 * 4096
    assert base >= 2 * 4 * nw + nw * 2 // 8 + 4096 * 64 * 4 and base < 2 * 4 * nw + nw // 4 + (8 << 20)
    assert lib.harp_calib_workspace_size(4096, 4096, 2, 4096, 4096, 1, 0, ctypes.byref(n)) == 0
    assert n.value - base == 2 * 4 * 4096 * 4096
    assert lib.harp_calib_workspace_size(4096, 4096, 2, 4096, 4096, 1, 1, ctypes.byref(n)) == 0
    assert n.value > base + 4 * 4 * nw
    assert lib.harp_calib_workspace_size(4096, 4096, 5, 4096, 4096, 0, 0, ctypes.byref(n)) == 1
    assert lib.harp_calib_workspace_size(4096, 4096, 2, 4096, 3000, 0, 0, ctypes.byref(n)) == 1
    assert lib.harp_calib_workspace_size(4096, 4096, 2, 4096, 4096, 0, 0, None) == 1


def _calib(lib, n_out, n_in, bits, group, w_in, w_out, W=FAKE, H=None, lam=0.0, loss=FAKE, ws=1 << 40):
    return lib.harp_calib_fit(n_out, n_in, bits, group, w_in, w_out, W, FAKE, FAKE, FAKE, FAKE, H, lam, loss, None,
                              None, FAKE, ws, None)


@pytest.mark.parametrize("n_out,n_in,bits,group,w_in,w_out,ws,err", [
    (4096, 4096, 2, 64, 4096, 4096, 1 << 20, 4),    # workspace too small
    (4096, 4096, 2, 32, 4096, 4096, 1 << 40, 2),    # unsupported group
    (4096, 4000, 2, 64, 4096, 4096, 1 << 40, 1),    # n_in not a multiple of 256
    (4000, 4096, 2, 64, 4096, 4096, 1 << 40, 1),    # n_out not a multiple of 32
    (65536, 4096, 2, 64, 4096, 4096, 1 << 40, 1),   # n_out is a butterfly batch: < 65536
    (4096, 4096, 2, 64, 3000, 4096, 1 << 40, 1),    # w_in not a power of two
    (4096, 11008, 2, 64, 4096, 4096, 1 << 40, 1),   # w_in does not divide n_in
])
def test_calib_rejects_bad_arguments(lib, n_out, n_in, bits, group, w_in, w_out, ws, err):
    st = _calib(lib, n_out, n_in, bits, group, w_in, w_out, ws=ws)
    assert st == err, lib.harp_last_error()


def test_calib_rejects_misaligned_pointers_and_negative_lambda(lib):
    assert _calib(lib, 4096, 4096, 2, 64, 4096, 4096, W=MIS) == 1
    assert _calib(lib, 4096, 4096, 2, 64, 4096, 4096, H=MIS) == 1
    assert _calib(lib, 4096, 4096, 2, 64, 4096, 4096, loss=None) == 1
    assert _calib(lib, 4096, 4096, 2, 64, 4096, 4096, lam=-1.0) == 1


def test_mr_plan_rejects_bad_arguments(lib):
    """Validation of the mixed-radix plan happens before any CUDA call."""
    h = ctypes.c_void_p()

    def create(d, radices, gauss=None, theta=FAKE):
        r = (ctypes.c_int * len(radices))(*radices)
        return lib.harp_mr_plan_create(ctypes.byref(h), d, len(radices), r, theta, FAKE, gauss, None)

    assert create(60, [3, 4, 5]) == 1            # odd radices without their Gaussian
    assert create(64, [8, 4]) == 1               # radices do not multiply to d
    assert create(128, [2, 64, 1]) == 1          # radix below 2
    assert create(16384 * 2, [128, 256]) == 1    # d too large, radices too large
    assert create(64, [8, 8], theta=MIS) == 1    # misaligned theta
    assert create(64, [8, 8], theta=None) == 1   # null theta
    assert not h.value
    assert lib.harp_mr_plan_destroy(None) == 0
    assert lib.harp_mr_butterfly_fwd(None, 1, FAKE, 0, FAKE, 0, None) == 1


def test_fault_hook_validates_and_switches_off(lib):
    """The testing hook of the failure paths takes no CUDA call: bad values are refused and
    the defaults switch it off again."""
    assert lib.harp_test_set_faults(-1, -1, -1) == 1
    assert lib.harp_test_set_faults(0, -2, -1) == 1
    assert lib.harp_test_set_faults(1000, 0, 3) == 0
    assert lib.harp_test_set_faults(0, -1, -1) == 0
