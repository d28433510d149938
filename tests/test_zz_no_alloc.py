"""df11_encode_static_ws: the encode entry point for callers that cannot
allocate device memory at the call site (a plugin inside another framework's
callback without its allocator, a process that reserved all device memory up
front).  It keeps its scratch in a fixed array inside the library instead of
taking a workspace.  Checked through the C ABI against df11_encode, the entry
point that takes a caller-provided workspace: every stored byte must match,
on two calls in a row (the second, smaller one runs over scratch left behind
by the first)."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def df11():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    import lossless_bf16_weight_df11_b200 as m
    return m


def _outputs(df11, sizes, dev):
    bufs = dict(
        stream=torch.empty(sizes.stream_alloc, dtype=torch.uint8, device=dev),
        gaps=torch.empty(sizes.gaps_alloc, dtype=torch.uint8, device=dev),
        block_pos=torch.empty(sizes.block_pos_alloc // 4, dtype=torch.int32, device=dev),
        sign_mantissa=torch.empty(sizes.sign_mantissa_alloc, dtype=torch.uint8, device=dev),
    )
    abi = df11.df11_encoded(stream=bufs["stream"].data_ptr(), gaps=bufs["gaps"].data_ptr(),
                            block_pos=bufs["block_pos"].data_ptr(),
                            sign_mantissa=bufs["sign_mantissa"].data_ptr())
    return bufs, abi


def _stored(bufs, sizes):
    return (bufs["stream"][: sizes.stream_bytes].cpu().numpy(),
            bufs["gaps"][: sizes.gaps_bytes].cpu().numpy(),
            bufs["block_pos"][: sizes.n_blocks + 1].cpu().numpy(),
            bufs["sign_mantissa"][: sizes.sign_mantissa_bytes].cpu().numpy())


def _encode_both(df11, x: np.ndarray, cap: int = 12):
    dev = torch.device("cuda", 0)
    w = torch.from_numpy(np.ascontiguousarray(x).reshape(-1).view(np.int16)).to(dev)
    n = w.numel()
    stream = torch.cuda.current_stream().cuda_stream
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    df11.check(df11.df11_histogram(w.data_ptr(), n, hist.data_ptr(), stream), "df11_histogram")
    h = hist.cpu().numpy().view(np.uint64)
    st, cb = df11.df11_build_codebook(h, cap)
    df11.check(st, "df11_build_codebook")
    st, sizes = df11.df11_encoded_sizes(cb, h, n)
    df11.check(st, "df11_encoded_sizes")

    ref, ref_abi = _outputs(df11, sizes, dev)
    ws = torch.empty(max(16, sizes.workspace_bytes), dtype=torch.uint8, device=dev)
    ref_status = torch.zeros(1, dtype=torch.int32, device=dev)
    df11.check(df11.df11_encode(w.data_ptr(), n, cb, sizes.total_bits, ref_abi, ws.data_ptr(),
                                ws.numel(), ref_status.data_ptr(), stream), "df11_encode")

    got, got_abi = _outputs(df11, sizes, dev)
    got_status = torch.zeros(1, dtype=torch.int32, device=dev)
    df11.check(df11.df11_encode_static_ws(w.data_ptr(), n, cb, sizes.total_bits, got_abi,
                                          got_status.data_ptr(), stream),
               "df11_encode_static_ws")
    torch.cuda.synchronize()
    assert int(ref_status.item()) == 0 and int(got_status.item()) == 0
    return _stored(ref, sizes), _stored(got, sizes)


def test_static_workspace_encode_matches_workspace_encode_twice(df11):
    first = workloads.matrix(2, 0)                    # 4096 x 4096, 4096 tiles
    second = workloads.random_bf16(1_000_003, seed=77)  # 245 tiles, ragged tail
    for x in (first, second):
        ref, got = _encode_both(df11, x)
        for name, a, b in zip(("stream", "gaps", "block_pos", "sign_mantissa"), ref, got):
            assert np.array_equal(a, b), f"{name} differs"


def test_static_workspace_encode_rejects_oversized_input(df11):
    dev = torch.device("cuda", 0)
    st, cb = df11.df11_build_codebook([0] * 127 + [1] + [0] * 128, 12)
    df11.check(st, "df11_build_codebook")
    small = torch.zeros(64, dtype=torch.uint8, device=dev)
    abi = df11.df11_encoded(stream=small.data_ptr(), gaps=small.data_ptr(),
                            block_pos=small.data_ptr(), sign_mantissa=small.data_ptr())
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    n = df11.STATIC_WS_MAX_N + 1
    st = df11.df11_encode_static_ws(small.data_ptr(), n, cb, n, abi, status.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert st == df11.DF11_ERR_TOO_LARGE


def test_static_workspace_encode_allocates_no_device_memory(df11):
    """With every buffer allocated beforehand and one warm-up call made (the
    first call on a device looks up the array's address and loads the
    kernels), a further call leaves the device's free memory unchanged."""
    dev = torch.device("cuda", 0)
    x = workloads.random_bf16(3_000_001, seed=78)
    w = torch.from_numpy(x.view(np.int16)).to(dev)
    n = w.numel()
    stream = torch.cuda.current_stream().cuda_stream
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    df11.check(df11.df11_histogram(w.data_ptr(), n, hist.data_ptr(), stream), "df11_histogram")
    h = hist.cpu().numpy().view(np.uint64)
    st, cb = df11.df11_build_codebook(h, 11)
    df11.check(st, "df11_build_codebook")
    st, sizes = df11.df11_encoded_sizes(cb, h, n)
    df11.check(st, "df11_encoded_sizes")
    bufs, abi = _outputs(df11, sizes, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        df11.check(df11.df11_encode_static_ws(w.data_ptr(), n, cb, sizes.total_bits, abi,
                                              status.data_ptr(), stream), "df11_encode_static_ws")
        torch.cuda.synchronize()

    call()
    free_before, _ = torch.cuda.mem_get_info(dev)
    call()
    free_after, _ = torch.cuda.mem_get_info(dev)
    assert free_after == free_before
    assert int(status.item()) == 0
