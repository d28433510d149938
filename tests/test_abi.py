"""CPU tests of the C-ABI library: it loads, exports every function
include/df11.h declares, and its host code (codebook, sizes, decode tables,
metadata validation) agrees with the oracle.  No GPU compute is called."""
import ctypes
import itertools

import numpy as np
import pytest

import lossless_bf16_weight_df11_b200 as df11
from lossless_bf16_weight_df11_b200 import build as df11_build
import oracle
import workloads


@pytest.fixture(scope="session")
def lib():
    df11_build.build()
    return df11.load()


def hist_from(counts, first=0):
    h = np.zeros(256, np.uint64)
    for i, c in enumerate(counts):
        h[first + i] = c
    return h


def test_exports_every_declared_symbol(lib):
    names = df11.declared_functions()
    assert {"df11_histogram", "df11_build_codebook", "df11_encode", "df11_decode",
            "df11_decode_block_batch", "df11_encoded_sizes", "df11_build_tables",
            "df11_validate", "df11_status_string", "df11_tables_bytes"} <= set(names)
    raw = ctypes.CDLL(df11.library_path())
    for name in names:
        assert hasattr(raw, name), name


def test_status_strings(lib):
    for s in range(8):
        assert df11.df11_status_string(s)
    assert df11.df11_status_string(0) == "ok"


def lib_codebook(h, cap=32):
    st, cb = df11.df11_build_codebook(h, cap)
    assert st == df11.DF11_OK
    return np.array(cb.len, np.uint8), np.array(cb.code, np.uint32), cb


def assert_same_codebook(h, cap=32):
    ln, code, cb = lib_codebook(h, cap)
    oln, ocode = oracle.codebook(h, cap)
    assert np.array_equal(ln, oln)
    assert np.array_equal(code, ocode)
    nz = oln[oln > 0]
    assert cb.n_symbols == nz.size
    if nz.size:
        assert cb.max_len == nz.max() and cb.min_len == nz.min()


@pytest.mark.parametrize("seed", range(300))
def test_codebook_matches_oracle_random(lib, seed):
    g = np.random.default_rng(seed)
    h = np.zeros(256, np.uint64)
    m = int(g.integers(1, 257))
    syms = g.choice(256, m, replace=False)
    kind = seed % 5
    if kind == 0:
        h[syms] = g.integers(1, 10, m)          # many ties
    elif kind == 1:
        h[syms] = g.integers(1, 1 << 40, m)     # huge counts
    elif kind == 2:
        h[syms] = g.geometric(0.3, m)           # skewed
    elif kind == 3:
        h[syms] = (2.0 ** g.uniform(0, 30, m)).astype(np.uint64)
    else:
        h[syms] = 7                             # all equal
    assert_same_codebook(h)


@pytest.mark.parametrize("cap", [8, 9, 10, 12, 16, 20, 24])
def test_codebook_matches_oracle_tight_caps(lib, cap):
    g = np.random.default_rng(cap)
    for _ in range(20):
        h = np.zeros(256, np.uint64)
        m = int(g.integers(2, min(256, 1 << cap) + 1))
        h[g.choice(256, m, replace=False)] = (2.0 ** g.uniform(0, 34, m)).astype(np.uint64) + 1
        assert_same_codebook(h, cap)


@pytest.mark.parametrize("k", [30, 33, 34, 35, 40, 45])
def test_codebook_matches_oracle_fibonacci(lib, k):
    h = hist_from(workloads.fibonacci_counts(k), first=60)
    assert_same_codebook(h, 32)
    ln, _, _ = lib_codebook(h, 32)
    assert ln.max() <= 32


def test_codebook_degenerate(lib):
    st, cb = df11.df11_build_codebook(np.zeros(256, np.uint64), 32)
    assert st == 0 and cb.n_symbols == 0
    ln, code, cb = lib_codebook(hist_from([5], first=200))
    assert ln[200] == 1 and code[200] == 0 and cb.n_symbols == 1
    ln, code, _ = lib_codebook(hist_from([5, 9], first=10))
    assert ln[10] == 1 and ln[11] == 1
    assert_same_codebook(np.full(256, 1 << 33, np.uint64))
    st, _ = df11.df11_build_codebook(np.ones(256, np.uint64), 7)  # 2^7 < 256 symbols
    assert st == df11.DF11_ERR_INVALID_ARG
    for cap in (0, 33):
        st, _ = df11.df11_build_codebook(np.ones(4, np.uint64), cap)
        assert st == df11.DF11_ERR_INVALID_ARG


@pytest.mark.parametrize("n", [0, 1, 9, 4097, 262_144])
def test_encoded_sizes_match_oracle(lib, n):
    x = workloads.random_bf16(n, seed=n)
    enc = oracle.encode(x)
    _, _, cb = lib_codebook(enc.hist)
    st, s = df11.df11_encoded_sizes(cb, enc.hist, n)
    assert st == 0
    assert s.total_bits == enc.total_bits and s.n_chunks == enc.n_chunks
    assert s.n_blocks == enc.n_blocks
    assert s.stream_bytes == enc.stream.size and s.gaps_bytes == enc.gaps_packed.size
    assert s.block_pos_bytes == 4 * enc.block_pos.size and s.sign_mantissa_bytes == n
    assert s.stored_bytes == oracle.stored_bytes(enc)
    assert s.stream_alloc >= s.stream_bytes + 16 and s.stream_alloc % 16 == 0
    assert s.gaps_alloc >= 160 * s.n_blocks and s.sign_mantissa_alloc % 16 == 0


def test_encoded_sizes_errors(lib):
    _, _, cb = lib_codebook(hist_from([3, 4], first=5))
    h = hist_from([3, 4, 1], first=5)
    st, _ = df11.df11_encoded_sizes(cb, h, 8)
    assert st == df11.DF11_ERR_SYMBOL_NOT_IN_CODEBOOK
    st, _ = df11.df11_encoded_sizes(cb, hist_from([3, 4], first=5), 1 << 33)
    assert st == df11.DF11_ERR_TOO_LARGE


def tables_of(cb):
    nb = df11.df11_tables_bytes()
    buf = np.zeros(nb, np.uint8)
    assert df11.df11_build_tables(cb, buf.ctypes.data, nb) == 0
    return buf


TABLE_BITS = df11.TABLE_BITS      # 11: the lookup table's window
LONG_FLAG = 1 << 26


def ror8(e: int) -> int:
    """The decoder's stored form of an exponent byte: rotated right by one bit."""
    return ((e >> 1) | (e << 7)) & 0xFF


def greedy_window(codes_by_str, bits):
    """Up to four whole codes from the left of a window string, with their starts."""
    out, starts, used = [], [], 0
    while len(out) < 4:
        found = None
        for L in range(1, len(bits) + 1 - used):
            s = bits[used:used + L]
            if s in codes_by_str:
                found = (codes_by_str[s], L)
                break
        if found is None:
            break
        out.append(found[0])
        starts.append(used)
        used += found[1]
    return out, starts, used


@pytest.mark.parametrize("which", ["workload1", "uniform", "fibonacci34", "two", "skew"])
def test_decode_table_against_oracle_codes(lib, which):
    """The library's decode tables describe the oracle's code: every window of
    the lookup table decodes, greedily, the codes the oracle's canonical code
    gives for those bits (at most four, with each one's start), and the
    long-code arrays decode every code canonically."""
    if which == "workload1":
        h = oracle.histogram(oracle.split(workloads.matrix(1, 0))[0])
    elif which == "uniform":
        h = np.ones(256, np.uint64)
    elif which == "fibonacci34":
        h = hist_from(workloads.fibonacci_counts(34), first=100)
    elif which == "two":
        h = hist_from([1, 1], first=0)
    else:
        h = hist_from([1000, 300, 100, 30, 10, 3, 1], first=120)
    ln, code, cb = lib_codebook(h)
    oln, ocode = oracle.codebook(h)
    codes_by_str = {format(int(ocode[s]), f"0{int(oln[s])}b"): s for s in range(256) if oln[s]}
    tab = tables_of(cb)
    K = TABLE_BITS
    lut = tab[: 8 << K].view(np.uint32).reshape(-1, 2)
    # the long-code arrays: limit u64[33], base u32[33], codelen u8[256], sym u8[256], then
    # max_len, min_len, n_symbols, lut_bits
    limit = tab[16384:16384 + 264].view(np.uint64)
    base = tab[16648:16648 + 132].view(np.uint32)
    codelen = tab[16780:16780 + 256]
    sym = tab[17036:17036 + 256]
    max_len, min_len, n_sym, lut_bits = tab[17292:17308].view(np.uint32)
    assert np.array_equal(codelen, oln)
    nz = oln[oln > 0]
    assert (max_len, min_len, n_sym, lut_bits) == (nz.max(), nz.min(), nz.size, K)
    for L in range(1, 33):
        at_L = [s_ for s_ in range(256) if oln[s_] == L]
        for s_ in at_L:   # canonical decoding of a long code: sym[code + base[L]]
            assert sym[(int(ocode[s_]) + int(base[L])) % 2 ** 32] == ror8(s_)
        if at_L:
            first = min(int(ocode[s_]) for s_ in at_L)
            assert int(limit[L]) == (first + len(at_L)) << (32 - L)
    for v in range(1 << K):
        syms, starts, used = greedy_window(codes_by_str, format(v, f"0{K}b"))
        x, c = int(lut[v, 0]), int(lut[v, 1])
        if not syms:
            # long-code flag; the window's bits counted as consumed, no codes
            assert x == 0 and c == (K << 28) | (0xFFF << 12) | LONG_FLAG, (v, hex(c))
            continue
        n = len(syms)
        fields = [starts[j] if j < n else 15 for j in (1, 2, 3)]
        assert c == (used << 28) | (n << 3) | (fields[0] << 12) | (fields[1] << 16) | \
            (fields[2] << 20), (v, hex(c))
        assert x == sum(ror8(s) << (8 * i) for i, s in enumerate(syms)), (v, hex(x))


def test_validate_accepts_oracle_metadata_and_rejects_corruption(lib):
    x = workloads.random_bf16(300_001, seed=5)
    enc = oracle.encode(x)
    min_len = int(enc.lengths[enc.lengths > 0].min())
    g = np.ascontiguousarray(enc.gaps_packed)
    pos = np.ascontiguousarray(enc.block_pos)

    def val(gaps=g, p=pos, n=enc.n, tb=enc.total_bits, ml=min_len):
        return df11.df11_validate(n, tb, ml, gaps.ctypes.data, gaps.size, p.ctypes.data, p.size)

    assert val() == 0
    bad = pos.copy(); bad[-1] += 1
    assert val(p=bad) == df11.DF11_ERR_CORRUPT
    bad = pos.copy(); bad[2], bad[3] = bad[3], bad[2]
    assert val(p=bad) == df11.DF11_ERR_CORRUPT
    bad = pos.copy(); bad[1] = bad[2]  # block 0 too large? still monotone -> count check
    bad[1] = 0
    assert val(p=bad) in (0, df11.DF11_ERR_CORRUPT)
    assert val(ml=33) == df11.DF11_ERR_INVALID_ARG
    assert val(n=1 << 33) == df11.DF11_ERR_TOO_LARGE
    assert val(tb=enc.total_bits + 64 * 300) == df11.DF11_ERR_INVALID_ARG  # too few gap bytes
    # a tail chunk whose gap points past the end of the stream
    C = enc.n_chunks
    tail = enc.gaps.copy()
    tail[-1] = min(31, enc.total_bits - 64 * (C - 1) + 1)
    if tail[-1] > enc.total_bits - 64 * (C - 1):
        gp = oracle.pack_gaps(tail)
        assert val(gaps=gp) == df11.DF11_ERR_CORRUPT


def test_sizes_from_bits_equal_encoded_sizes():
    g = np.random.default_rng(8)
    for _ in range(200):
        h = np.zeros(256, np.uint64)
        m = int(g.integers(1, 257))
        h[g.choice(256, m, replace=False)] = g.integers(1, 10 ** int(g.integers(1, 6)), m)
        st, cb = df11.df11_build_codebook(h, int(g.integers(8, 33)))
        if st:
            continue
        n = int(h.sum())
        st, a = df11.df11_encoded_sizes(cb, h, n)
        assert st == df11.DF11_OK
        st, b = df11.df11_sizes_from_bits(n, a.total_bits)
        assert st == df11.DF11_OK
        assert bytes(a) == bytes(b)
    assert df11.df11_sizes_from_bits(10, 9)[0] == df11.DF11_ERR_INVALID_ARG     # < 1 bit a value
    assert df11.df11_sizes_from_bits(10, 321)[0] == df11.DF11_ERR_INVALID_ARG   # > 32 bits a value
    assert df11.df11_sizes_from_bits(2 ** 32, 2 ** 33)[0] == df11.DF11_ERR_TOO_LARGE
    assert df11.df11_sizes_from_bits(0, 0)[0] == df11.DF11_OK


def test_device_codebook_launchers_check_arguments_first():
    """Argument errors are returned before any device query."""
    assert df11.df11_build_codebook_device(0, 12, 16, 16, 16, 0, 0) == df11.DF11_ERR_INVALID_ARG
    assert df11.df11_build_codebook_device(16, 0, 16, 16, 16, 0, 0) == df11.DF11_ERR_INVALID_ARG
    assert df11.df11_build_codebook_device(16, 33, 16, 16, 16, 0, 0) == df11.DF11_ERR_INVALID_ARG
    assert df11.df11_build_codebook_device(16, 12, 16, 24, 16, 0, 0) == df11.DF11_ERR_INVALID_ARG
    out = df11.df11_encoded(stream=16, gaps=16, block_pos=16, sign_mantissa=16, block_max=0)
    assert df11.df11_encode_device_codebook(16, 100, 0, 300, out, 16, 4096, 16, 0) == \
        df11.DF11_ERR_INVALID_ARG
    assert df11.df11_encode_device_codebook(16, 100, 18, 300, out, 16, 4096, 16, 0) == \
        df11.DF11_ERR_INVALID_ARG
    assert df11.df11_encode_device_codebook(16, 100, 16, 99, out, 16, 4096, 16, 0) == \
        df11.DF11_ERR_INVALID_ARG
    assert df11.df11_encode_device_codebook(16, 2 ** 33, 16, 2 ** 34, out, 16, 4096, 16, 0) == \
        df11.DF11_ERR_TOO_LARGE


def test_shared_codebook_code_matches_the_oracle_when_the_cap_binds():
    """The host builder (shared with the device kernel) against the oracle on
    Fibonacci counts at every cap from the smallest feasible to 32."""
    f = workloads.fibonacci_counts(34)
    h = hist_from(f, first=50)
    for cap in range(6, 33):
        assert_same_codebook(h, cap)
