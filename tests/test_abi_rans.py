"""CPU tests of the rANS variant's host code in the C-ABI library: the
frequencies agree with the oracle's, and the device tables hold what
include/df11_rans.h says they hold.  No GPU compute is called."""
import numpy as np
import pytest

import lossless_bf16_weight_df11_b200 as df11
from lossless_bf16_weight_df11_b200 import build as df11_build
import oracle
import workloads


@pytest.fixture(scope="module", autouse=True)
def lib():
    df11_build.build()
    return df11.load()


def random_hist(g, rare: bool) -> np.ndarray:
    h = np.zeros(256, np.uint64)
    m = int(g.integers(1, 257))
    h[g.choice(256, m, replace=False)] = g.integers(1, 10 ** int(g.integers(1, 7)), m).astype(np.uint64)
    if rare:
        h[g.choice(256, min(m, 5), replace=False)] = 1
    return h


def test_frequencies_match_the_oracle():
    g = np.random.default_rng(21)
    for t in range(2000):
        h = random_hist(g, rare=t % 3 == 0)
        st, f = df11.df11_rans_freqs(h)
        assert st == df11.DF11_OK
        assert f == oracle.rans_freqs(h).tolist()


def test_frequencies_of_the_workloads_match_the_oracle():
    for wl, idx in [(1, 0), (2, 0), (5, 4)]:
        x = workloads.matrix(wl, idx).reshape(-1)[: 1 << 20]
        h = oracle.histogram(oracle.split(x)[0])
        st, f = df11.df11_rans_freqs(h)
        assert st == df11.DF11_OK and f == oracle.rans_freqs(h).tolist()
    for x in (workloads.all_patterns(), workloads.fibonacci_exponents(30)[:100_000]):
        h = oracle.histogram(oracle.split(x)[0])
        assert df11.df11_rans_freqs(h)[1] == oracle.rans_freqs(h).tolist()


def test_frequencies_edge_cases():
    st, f = df11.df11_rans_freqs(np.zeros(256, np.uint64))
    assert st == df11.DF11_OK and sum(f) == 0
    h = np.zeros(256, np.uint64)
    h[77] = 5
    assert df11.df11_rans_freqs(h)[1][77] == 4096
    h = np.full(256, 2 ** 24 + 1, np.uint64)      # n > 2^32: more than one matrix may hold
    assert df11.df11_rans_freqs(h)[0] == df11.DF11_ERR_TOO_LARGE


def tables_of(freq):
    host = np.zeros(df11.RANS_TABLES_BYTES, np.uint8)
    st = df11.df11_rans_build_tables(freq, host.ctypes.data, host.size)
    return st, host.view(np.uint32)


def test_tables_follow_the_header_layout():
    g = np.random.default_rng(5)
    for _ in range(50):
        h = random_hist(g, rare=True)
        f = oracle.rans_freqs(h)
        st, t = tables_of(f)
        assert st == df11.DF11_OK
        slot, enc = t[:4096], t[4096:]
        cum = np.concatenate([[0], np.cumsum(f)[:-1]]).astype(np.int64)
        for s in np.flatnonzero(f):
            assert enc[s] == int(f[s]) | (int(cum[s]) << 16)
            e = slot[cum[s]: cum[s] + f[s]]
            assert np.all(e & 0xFF == s)
            assert np.array_equal((e >> 8) & 0xFFF, np.arange(f[s]))
            assert np.all((e >> 20) + 1 == f[s])
        assert np.all(enc[f == 0] == 0)
        # decoding identity for every slot and a few states:
        # x' = f * (x >> 12) + (slot - cum) must invert the encoder's step
        for x in (1 << 16, 123_456_789, (1 << 32) - 1):
            sl = x & 4095
            e = int(slot[sl])
            s, bias, fs = e & 0xFF, (e >> 8) & 0xFFF, (e >> 20) + 1
            xd = fs * (x >> 12) + bias
            assert (xd // fs) * 4096 + xd % fs + int(cum[s]) == x


def test_tables_reject_bad_sums():
    f = np.zeros(256, np.uint32)
    f[3] = 4095
    assert tables_of(f)[0] == df11.DF11_ERR_INVALID_ARG
    f[4] = 2
    assert tables_of(f)[0] == df11.DF11_ERR_INVALID_ARG
    st, t = tables_of(np.zeros(256, np.uint32))
    assert st == df11.DF11_OK and not t.any()
    host = np.zeros(100, np.uint8)
    assert df11.df11_rans_build_tables(oracle.rans_freqs(np.ones(256, np.uint64)), host.ctypes.data,
                                       host.size) == df11.DF11_ERR_INVALID_ARG


def test_units():
    for n, u in [(0, 0), (1, 1), (16384, 1), (16385, 2), (2 ** 32 - 1, 262144)]:
        assert df11.df11_rans_units(n) == u


def test_launchers_reject_bad_arguments_without_a_device():
    """Argument checks run before any device query."""
    assert df11.df11_rans_encode_sizes(0, 10, 0, 0, 0, 0, 0) == df11.DF11_ERR_INVALID_ARG
    assert df11.df11_rans_encode_sizes(16, 2 ** 32, 16, 16, 16, 0, 0) == df11.DF11_ERR_TOO_LARGE
    assert df11.df11_rans_encode(8, 10, 16, 16, 16, 16, 16, 0, 0) == df11.DF11_ERR_INVALID_ARG
    m = df11.df11_rans_matrix(n=100, stream=16, off16=16, sign_mantissa=24, tables=16)
    assert df11.df11_rans_decode_batch([m], [16], 0, 0) == df11.DF11_ERR_INVALID_ARG
    m = df11.df11_rans_matrix(n=2 ** 33, stream=16, off16=16, sign_mantissa=16, tables=16)
    assert df11.df11_rans_decode_batch([m], [16], 0, 0) == df11.DF11_ERR_TOO_LARGE
