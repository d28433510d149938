"""The codebook built on the device (df11_build_codebook_device) against the
host's (df11_build_codebook + df11_build_tables + df11_encoded_sizes) and the
oracle's, and the all-device compressor (codec.compress_block_device)
against compress_block.

Histograms are uploaded as they are: random ones of every size of alphabet,
Fibonacci counts (the length cap binds and package-merge runs), a single
exponent, none at all, and all 256 exponents under a cap too small for them."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

GUARD = 256
PATTERN = 0xA5


@pytest.fixture(scope="module")
def df11():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    import lossless_bf16_weight_df11_b200 as m
    return m


@pytest.fixture(scope="module")
def codec(df11):
    import lossless_bf16_weight_df11_b200.codec as c
    return c


def guarded(nbytes):
    full = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    return full, full[GUARD:GUARD + nbytes]


def intact(full, nbytes):
    f = full.cpu().numpy()
    return bool((f[:GUARD] == PATTERN).all() and (f[GUARD + nbytes:] == PATTERN).all())


def device_codebook(df11, hist, cap):
    nt = df11.df11_tables_bytes()
    h = torch.from_numpy(np.ascontiguousarray(hist, np.uint64).view(np.int64)).cuda()
    cb_full, cb = guarded(df11.CODEBOOK_BYTES)
    t_full, tab = guarded(nt)
    b_full, bits = guarded(8)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.check(df11.df11_build_codebook_device(h.data_ptr(), cap, cb.data_ptr(), tab.data_ptr(),
                                               bits.data_ptr(), status.data_ptr(), 0))
    torch.cuda.synchronize()
    assert intact(cb_full, df11.CODEBOOK_BYTES) and intact(t_full, nt) and intact(b_full, 8)
    return (int(status.item()), cb.cpu().numpy(), tab.cpu().numpy(),
            int(bits.cpu().numpy().view(np.uint64)[0]))


def host_codebook(df11, hist, cap):
    st, cb = df11.df11_build_codebook(hist, cap)
    if st:
        return st, None, None, None
    host = np.zeros(df11.df11_tables_bytes(), np.uint8)
    df11.check(df11.df11_build_tables(cb, host.ctypes.data, host.size))
    n = int(np.asarray(hist, np.uint64).sum())
    st, sizes = df11.df11_encoded_sizes(cb, hist, n)
    df11.check(st)
    return 0, np.frombuffer(bytes(cb), np.uint8), host, int(sizes.total_bits)


def histograms():
    g = np.random.default_rng(77)
    out = []
    for m in (1, 2, 3, 5, 17, 64, 200, 256):
        for _ in range(3):
            h = np.zeros(256, np.uint64)
            h[g.choice(256, m, replace=False)] = g.integers(1, 10 ** int(g.integers(1, 7)), m)
            out.append((f"random_{m}", h, 32))
            out.append((f"random_{m}_cap11", h, 11))
    fib = np.zeros(256, np.uint64)
    fib[50:50 + 34] = workloads.fibonacci_counts(34)
    out += [("fibonacci_cap32", fib, 32), ("fibonacci_cap12", fib, 12), ("fibonacci_cap11", fib, 11),
            ("fibonacci_cap6", fib, 6)]
    one = np.zeros(256, np.uint64)
    one[127] = 1000
    out += [("one_symbol", one, 11), ("empty", np.zeros(256, np.uint64), 11),
            ("all_equal_cap8", np.full(256, 9, np.uint64), 8)]
    x = workloads.matrix(2, 0).reshape(-1)
    out.append(("matrix_4096x4096", oracle.histogram(oracle.split(x)[0]), 11))
    return out


@pytest.mark.parametrize("name,hist,cap", histograms(), ids=[h[0] for h in histograms()])
def test_device_codebook_equals_host_and_oracle(df11, name, hist, cap):
    st_d, cb_d, tab_d, bits_d = device_codebook(df11, hist, cap)
    st_h, cb_h, tab_h, bits_h = host_codebook(df11, hist, cap)
    assert st_d == st_h == 0
    assert np.array_equal(cb_d, cb_h)
    assert np.array_equal(tab_d, tab_h)
    assert bits_d == bits_h
    ln, code = oracle.codebook(hist, cap)
    cb = df11.df11_codebook.from_buffer_copy(cb_d.tobytes())
    assert list(cb.len) == ln.tolist() and list(cb.code) == code.tolist()


def test_cap_too_small_is_reported_and_nothing_written(df11):
    st, cb, tab, bits = device_codebook(df11, np.full(256, 3, np.uint64), 7)
    assert st == df11.DF11_ERR_INVALID_ARG
    assert (cb == PATTERN).all() and (tab == PATTERN).all()


def to_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda()


def test_device_compressor_equals_compress_block(codec):
    names = workloads.WORKLOADS[3][1]
    xs = [workloads.matrix(3, i).reshape(-1) for i in range(len(names))]
    xs += [workloads.fibonacci_exponents(30)[:300_000], workloads.constant(5000, 0x3F80),
           workloads.random_bf16(17, seed=3), workloads.all_patterns()]
    ws = [to_dev(x) for x in xs]
    for cap in (11, 32):
        a = codec.compress_block(ws, cap=cap)
        b = codec.compress_block_device(ws, cap=cap)
        for ma, mb, x in zip(a, b, xs):
            assert bytes(ma.codebook) == bytes(mb.codebook)
            assert ma.total_bits == mb.total_bits and ma.max_block_codes == mb.max_block_codes
            ha, hb = ma.host_arrays(), mb.host_arrays()   # the stored bytes (no padding)
            for k in ha:
                assert np.array_equal(ha[k], hb[k]), k
            assert torch.equal(ma.tables, mb.tables)
            assert np.array_equal(ma.hist, mb.hist)
        outs = codec.decompress_block(b)
        for o, w in zip(outs, ws):
            assert torch.equal(o.reshape(-1).view(torch.int16), w)


def test_device_codebook_encode_reports_inconsistent_bits(df11, codec):
    """df11_encode_device_codebook checks total_bits on the device."""
    x = workloads.random_bf16(100_000, seed=4)
    w = to_dev(x)
    m = codec.compress_block_device([w])[0]
    meta = torch.zeros(1312, dtype=torch.uint8, device="cuda")
    meta[:df11.CODEBOOK_BYTES] = torch.from_numpy(
        np.frombuffer(bytes(m.codebook), np.uint8).copy()).cuda()
    st, sizes = df11.df11_sizes_from_bits(m.n, m.total_bits + 64)
    df11.check(st)
    bufs = codec.alloc_encoded(sizes, w.device)
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    ws = torch.empty(sizes.workspace_bytes, dtype=torch.uint8, device="cuda")
    out = df11.df11_encoded(stream=bufs["stream"].data_ptr(), gaps=bufs["gaps"].data_ptr(),
                            block_pos=bufs["block_pos"].data_ptr(),
                            sign_mantissa=bufs["sign_mantissa"].data_ptr(),
                            block_max=status.data_ptr() + 4)
    df11.check(df11.df11_encode_device_codebook(w.data_ptr(), m.n, meta.data_ptr(),
                                                m.total_bits + 64, out, ws.data_ptr(), ws.numel(),
                                                status.data_ptr(), 0))
    torch.cuda.synchronize()
    assert int(status[0].item()) == df11.DF11_ERR_CORRUPT
