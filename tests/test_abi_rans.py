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


def validate(enc, stream=None, off16=None, n=None):
    s = np.ascontiguousarray(enc.stream if stream is None else stream, np.uint8)
    o = np.ascontiguousarray(enc.off16 if off16 is None else off16, np.uint32)
    return df11.df11_rans_validate(enc.n if n is None else n, s.ctypes.data, s.size,
                                   o.ctypes.data, o.size)


@pytest.mark.parametrize("n", [0, 1, 31, 16384, 16385, 100_003])
def test_validate_accepts_the_oracle_encoding(n):
    enc = oracle.rans_encode(workloads.random_bf16(n, seed=n + 3))
    assert validate(enc) == df11.DF11_OK


def test_validate_accepts_edge_encodings():
    for x in (workloads.constant(70_000, 0x3F80), workloads.shuffled_patterns(copies=1, seed=2),
              workloads.fibonacci_exponents(30)[:50_000]):
        assert validate(oracle.rans_encode(x)) == df11.DF11_OK


def test_validate_rejects_corrupt_metadata():
    enc = oracle.rans_encode(workloads.random_bf16(3 * 16384 + 100, seed=7))
    u1 = 16 * int(enc.off16[1])

    def stream_with(pos, value, width=1):
        s = enc.stream.copy()
        s[pos:pos + width] = np.frombuffer(int(value).to_bytes(width, "little"), np.uint8)
        return s

    off = enc.off16.copy()
    off[2], off[1] = off[1], off[2]                  # decreasing offsets
    assert validate(enc, off16=off) == df11.DF11_ERR_CORRUPT
    off = enc.off16.copy()
    off[-1] += 1                                      # last offset past the stream
    assert validate(enc, off16=off) == df11.DF11_ERR_CORRUPT
    off = enc.off16.copy()
    off[1] = off[0] + 8                               # a unit smaller than its header
    off[2] = max(off[2], off[1])
    assert validate(enc, off16=off) == df11.DF11_ERR_CORRUPT
    off = enc.off16.copy()
    off[1] = off[-1] + 100                            # an offset beyond the end (read guard)
    assert validate(enc, off16=off) == df11.DF11_ERR_CORRUPT
    assert validate(enc, stream=stream_with(u1 + 128, 3, 2)) == df11.DF11_ERR_CORRUPT   # start[0]
    assert validate(enc, stream=stream_with(u1 + 130, 0xFFFF, 2)) == df11.DF11_ERR_CORRUPT
    assert validate(enc, stream=stream_with(u1 + 4 * 9, 0x1234, 4)) == df11.DF11_ERR_CORRUPT
    # a last unit of 20 values: lanes 20..31 code nothing, so their states must be exactly 2^16
    tail = oracle.rans_encode(workloads.random_bf16(3 * 16384 + 20, seed=8))
    last = 16 * int(tail.off16[3])
    s = tail.stream.copy()
    s[last + 4 * 31: last + 4 * 32] = np.frombuffer(((1 << 16) + 1).to_bytes(4, "little"), np.uint8)
    assert validate(tail) == df11.DF11_OK
    assert validate(tail, stream=s) == df11.DF11_ERR_CORRUPT
    assert validate(enc, off16=enc.off16[:-1]) == df11.DF11_ERR_INVALID_ARG
    assert validate(enc, n=2 ** 33) == df11.DF11_ERR_TOO_LARGE
