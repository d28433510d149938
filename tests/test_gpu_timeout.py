"""A bounded wait inside the decode kernel runs out: the kernel reports
DF11_ERR_TIMEOUT through its status word, writes nothing outside its output,
leaves no copy of its own in flight, and the GPU goes on decoding correctly.

The failure is made without any fault: the test build of the library
(libdf11_b200_test.so, the same sources compiled with DF11_TEST_HOOKS and a
wait limit of 256 polls) has one extra entry point, df11_test_decode_starved,
whose stream-stage barriers each expect 16 bytes more than their bulk copies
deliver.  Every copy lands in full, but no stage barrier ever completes, so
every bounded wait on one gives up.  The product library has neither the hook
nor the entry point.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

DF11_ERR_TIMEOUT = 6
GUARD = 4096
PATTERN = 0xA5


@pytest.fixture(scope="module")
def libs():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    path = build.build_test()
    import lossless_bf16_weight_df11_b200 as df11
    import lossless_bf16_weight_df11_b200.codec as codec
    test_lib = ctypes.CDLL(path)
    fn = test_lib.df11_test_decode_starved
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(df11.df11_matrix), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p]
    return df11, codec, fn


def test_product_library_has_no_test_hook(libs):
    df11, _, _ = libs
    assert not hasattr(df11.load(), "df11_test_decode_starved")


@pytest.mark.parametrize("n", [4_097, 3_000_001])
def test_starved_wait_reports_timeout_then_decode_recovers(libs, n):
    df11, codec, starved = libs
    x = workloads.random_bf16(n, seed=600 + n)
    w = torch.from_numpy(x.view(np.int16)).cuda()
    m = codec.compress(w)
    full = torch.full((2 * n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    out = full[GUARD:GUARD + 2 * n]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = starved(ctypes.byref(m.abi()), out.data_ptr(), status.data_ptr(),
                 int(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()   # the kernel returned: every wait was bounded
    assert int(status.item()) == DF11_ERR_TIMEOUT
    f = full.cpu().numpy()
    assert (f[:GUARD] == PATTERN).all() and (f[GUARD + 2 * n:] == PATTERN).all()
    # the device is still usable: a normal decode of the same matrix is exact
    status.zero_()
    got = codec.decompress(m, status=status)
    assert int(status.item()) == 0
    assert np.array_equal(got.reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16), x)
