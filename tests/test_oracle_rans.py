"""Pins for the oracle's rANS exponent-codec variant (a comparison codec for the
Huffman exponent coding; the DFloat11 page's discussion names rANS, and the
coding step is range ANS as Duda (2013) defines it).  Each test checks the
oracle against something other than itself: hand-derived streams, the
largest-remainder apportionment the frequency reading restates, closed forms
(one symbol; uniform frequencies, where rANS is a fixed 8-bit code), the
information bound of the coding step, and brute force over tiny inputs.
No GPU is needed."""
import itertools
import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
M = 4096


def hist_of(counts: dict) -> np.ndarray:
    h = np.zeros(256, np.uint64)
    for s, c in counts.items():
        h[int(s)] = c
    return h


def weights_with_exponents(e) -> np.ndarray:
    """BF16 words with the given exponents; sign and mantissa vary by index."""
    e = np.asarray(e, np.uint32)
    i = np.arange(e.size, dtype=np.uint32)
    return (((i & 1) << 15) | (e << 7) | (i * 37 % 128)).astype(np.uint16)


def freq_array(d: dict) -> np.ndarray:
    f = np.zeros(256, np.uint32)
    for s, v in d.items():
        f[int(s)] = v
    return f


def golden_cases():
    return json.load(open(os.path.join(GOLDEN, "rans_tiny.json")))["cases"]


def unit_bytes_from_fields(case) -> bytes:
    b = b"".join(struct.pack("<I", int(h, 16)) for h in case["states_hex"])
    b += b"".join(struct.pack("<H", v) for v in case["segment_starts"])
    b += b"".join(struct.pack("<H", int(h, 16)) for h in case["words_hex"])
    return b + bytes(case["unit_bytes"] - len(b))


def golden_exponents(case) -> np.ndarray:
    if "exponents" in case:
        return np.array(case["exponents"], np.uint32)
    e = np.full(65, 127, np.uint32)
    e[0], e[32], e[64] = 128, 128, 129
    return e


# ---- Q1: frequencies ------------------------------------------------------

@pytest.mark.parametrize("counts,want", [
    ({10: 1, 11: 1}, {10: 2048, 11: 2048}),
    ({0: 3, 1: 1}, {0: 3072, 1: 1024}),
    # floor(4096/3) = 1365, floor(8192/3) = 2730, sum 4095; deficits 1 and 2 -> +1 to symbol 6
    ({5: 1, 6: 2}, {5: 1365, 6: 2731}),
    # three equal counts: 1365 each, one short, equal deficits -> the smallest symbol
    ({0: 1, 1: 1, 2: 1}, {0: 1366, 1: 1365, 2: 1365}),
    # floor(4096*10^6/(10^6+1)) = 4095; the rare symbol is raised to 1; sum 4096
    ({0: 10**6, 1: 1}, {0: 4095, 1: 1}),
    # 100 rare symbols at 1 each and 4095 for the common one: 99 too many, all taken from it
    ({0: 10**6, **{s: 1 for s in range(1, 101)}}, {0: 3996, **{s: 1 for s in range(1, 101)}}),
    ({200: 7}, {200: 4096}),
    ({}, {}),
])
def test_frequencies_hand_examples(counts, want):
    f = oracle.rans_freqs(hist_of(counts))
    assert {s: int(f[s]) for s in range(256) if f[s]} == want


def test_frequencies_are_the_largest_remainder_apportionment():
    """Where no symbol needs raising to 1, the reading is Hamilton's
    largest-remainder method: each f is floor(c*M/n) or one more, and the
    symbols that get one more are those with the largest remainders."""
    g = np.random.default_rng(3)
    for trial in range(40):
        m = int(g.integers(2, 60))
        syms = g.choice(256, m, replace=False)
        h = np.zeros(256, np.uint64)
        h[syms] = g.integers(1000, 10**6, m).astype(np.uint64)
        n = int(h.sum())
        if any(int(h[s]) * M < n for s in syms):
            continue
        f = oracle.rans_freqs(h)
        assert int(f.sum()) == M
        quota = {int(s): Fraction(int(h[s]) * M, n) for s in syms}
        base = {s: math.floor(q) for s, q in quota.items()}
        extra = M - sum(base.values())
        order = sorted(quota, key=lambda s: (-(quota[s] - base[s]), s))
        want = {s: base[s] + (1 if s in order[:extra] else 0) for s in quota}
        assert {s: int(f[s]) for s in quota} == want
        assert all(f[s] == 0 for s in range(256) if h[s] == 0)


def test_frequencies_sum_and_support():
    g = np.random.default_rng(4)
    for _ in range(60):
        h = np.zeros(256, np.uint64)
        m = int(g.integers(1, 256))
        h[g.choice(256, m, replace=False)] = g.integers(1, 10**7, m).astype(np.uint64)
        f = oracle.rans_freqs(h)
        assert int(f.sum()) == M
        assert np.array_equal(f > 0, h > 0)


# ---- Q2-Q4: hand-derived streams ------------------------------------------

@pytest.mark.parametrize("case", golden_cases(), ids=lambda c: c["name"])
def test_golden_stream(case):
    e = golden_exponents(case)
    w = weights_with_exponents(e)
    freq = freq_array(case["freq"])
    if case["name"] == "two_values_data_frequencies":
        assert np.array_equal(oracle.rans_freqs(oracle.histogram(e.astype(np.uint8))), freq)
        enc = oracle.rans_encode(w)
    else:
        enc = oracle.rans_encode(w, freq=freq)
    assert enc.stream.tobytes() == unit_bytes_from_fields(case)
    assert enc.off16.tolist() == case["off16"]
    assert np.array_equal(oracle.rans_decode(enc), w)


# ---- closed forms ----------------------------------------------------------

def test_single_symbol_costs_only_headers():
    """f = M: the coding step is the identity, so no unit emits a word and
    every state stays at 2^16."""
    n = 3 * 16384 + 5
    w = workloads.constant(n, 0x3F80)
    enc = oracle.rans_encode(w)
    unit = struct.pack("<I", 1 << 16) * 32 + bytes(16)
    assert enc.stream.tobytes() == unit * 4
    assert enc.off16.tolist() == [0, 9, 18, 27, 36]
    assert np.array_equal(oracle.rans_decode(enc), w)


def lane_lengths(n: int):
    """Values each state of each unit codes (value u*16384 + 32k + l -> lane l)."""
    out = []
    for u in range((n + 16383) // 16384):
        m = min(16384, n - u * 16384)
        out.append([(m - l + 31) // 32 if l < m else 0 for l in range(32)])
    return out


def test_uniform_frequencies_are_a_fixed_8_bit_code():
    """Every exponent equally often -> f = 16 = M / 2^8 for all 256 symbols.
    Then each symbol adds exactly 8 bits to the state and a renormalisation
    removes exactly 16: from 2^16 (17 bits) the state goes 17 -> 25 bits,
    then (at >= 2^24 = 16 << 20) emits and drops to 9 bits before the next
    symbol takes it back to 17.  A lane that codes m values emits
    floor(m / 2) words and ends with 17 bits (m even) or 25 bits (m odd);
    cum[s] = 16 s, so the final state's slot (x mod M) lies in [16 s, 16 s +
    16) for the symbol s of the lane's first value, the first one decoded."""
    full = workloads.shuffled_patterns(copies=1, seed=11)    # 65536 values, 256 of each exponent
    assert set(oracle.rans_encode(full).freq.tolist()) == {16}
    # the same frequencies given for a ragged prefix: lanes of odd and even length
    for x in (full, full[: 3 * 16384 + 77]):
        enc = oracle.rans_encode(x, freq=np.full(256, 16, np.uint32))
        e, _ = oracle.split(x)
        for u, lens in enumerate(lane_lengths(x.size)):
            p = enc.stream[16 * enc.off16[u]: 16 * enc.off16[u + 1]].tobytes()
            states = struct.unpack("<32I", p[:128])
            words = sum(m // 2 for m in lens)
            assert 144 + 2 * words <= len(p) < 144 + 2 * words + 16
            for l, (m, st) in enumerate(zip(lens, states)):
                if m == 0:
                    assert st == 1 << 16
                    continue
                if m % 2 == 0:
                    assert 1 << 16 <= st < 1 << 17
                else:
                    assert 1 << 24 <= st < 1 << 25
                assert (st % M) >> 4 == e[u * 16384 + l]
        assert np.array_equal(oracle.rans_decode(enc), x)


def test_size_within_the_coding_step_bounds():
    """Each coding step maps x (at least 16 f after renormalisation) to x' with
    floor(x/f) M <= x' < (floor(x/f) + 1) M, so log2 x' - log2 x lies within
    log2(M/f) + [log2(15/16), log2(17/16)]; a renormalisation removes 16
    bits and at most one word.  Summed over a unit, the bits held (16 per
    word plus log2 of the final states, less the 32 * 16 bits of the initial
    states) are bounded by the information content sum log2(M/f)."""
    x = workloads.matrix(1, 0).reshape(-1)[: 5 * 16384 + 77]
    enc = oracle.rans_encode(x)
    e, _ = oracle.split(x)
    info = np.log2(M / enc.freq[e].astype(np.float64))
    for u, lens in enumerate(lane_lengths(x.size)):
        p = enc.stream[16 * enc.off16[u]: 16 * enc.off16[u + 1]].tobytes()
        states = struct.unpack("<32I", p[:128])
        starts = struct.unpack("<8H", p[128:144])
        n_words = (len(p) - 144) // 2
        while n_words and p[144 + 2 * n_words - 2: 144 + 2 * n_words] == b"\0\0":
            n_words -= 1          # a trailing zero word is padding or a real zero: bound both ways
        held = 16 * n_words + sum(math.log2(s) for s in states) - 32 * 16
        lo_i, hi_i = u * 16384, min(x.size, (u + 1) * 16384)
        total = float(info[lo_i:hi_i].sum())
        k = hi_i - lo_i
        assert total + k * math.log2(15 / 16) - 16 <= held <= total + k * math.log2(17 / 16) + 16
        # held bits are close to the information in practice (well inside the bound)
        assert abs(held - total) < 0.01 * k + 64
        assert starts[0] == 0 and list(starts) == sorted(starts)


# ---- brute force and round trips -------------------------------------------

def test_brute_force_tiny_inputs_are_injective_and_round_trip():
    """All 3^4 exponent sequences of 4 values over 3 symbols, with fixed
    frequencies 4000/64/32, at lanes 0..3 of one unit, and all 3^3
    sequences of one lane (values 0, 32, 64 of a 65-value input)."""
    freq = freq_array({100: 4000, 101: 64, 102: 32})
    seen = set()
    for seq in itertools.product((100, 101, 102), repeat=4):
        w = weights_with_exponents(seq)
        enc = oracle.rans_encode(w, freq=freq)
        assert np.array_equal(oracle.rans_decode(enc), w)
        seen.add(enc.stream.tobytes())
    assert len(seen) == 81
    seen = set()
    for seq in itertools.product((100, 101, 102), repeat=3):
        e = np.full(65, 100, np.uint32)
        e[0], e[32], e[64] = seq
        w = weights_with_exponents(e)
        enc = oracle.rans_encode(w, freq=freq)
        assert np.array_equal(oracle.rans_decode(enc), w)
        seen.add(enc.stream.tobytes())
    assert len(seen) == 27


@pytest.mark.parametrize("n", [0, 1, 31, 32, 33, 2047, 2048, 16383, 16384, 16385, 100_003])
def test_round_trip_edge_sizes(n):
    x = workloads.random_bf16(n, seed=n + 1)
    enc = oracle.rans_encode(x)
    assert enc.units == (n + 16383) // 16384 == enc.off16.size - 1
    assert np.array_equal(oracle.rans_decode(enc), x)


def test_round_trip_long_codes_and_all_patterns():
    for x in (workloads.fibonacci_exponents(30)[:200_000], workloads.all_patterns()):
        enc = oracle.rans_encode(x)
        assert np.array_equal(oracle.rans_decode(enc), x)


def test_symbol_without_frequency_is_rejected():
    w = weights_with_exponents([127, 128, 129])
    with pytest.raises(ValueError):
        oracle.rans_encode(w, freq=freq_array({127: 2048, 128: 2048}))


@pytest.mark.parametrize("where", ["state", "word", "segment_start"])
def test_corruption_is_detected(where):
    x = workloads.random_bf16(40_000, seed=17)
    enc = oracle.rans_encode(x)
    p = 16 * int(enc.off16[1])           # unit 1
    s = enc.stream.copy()
    if where == "state":
        s[p + 4 * 5] ^= 0x01
    elif where == "word":
        s[p + 144 + 2 * 10] ^= 0x40
    else:
        s[p + 128 + 2 * 3] ^= 0x01
    bad = oracle.RansEncoded(n=enc.n, hist=enc.hist, freq=enc.freq, stream=s, off16=enc.off16,
                             sign_mantissa=enc.sign_mantissa)
    try:
        y = oracle.rans_decode(bad)
    except ValueError:
        return
    assert not np.array_equal(y, x)     # never a silent wrong-but-equal result
    pytest.fail("corruption decoded without an error")


def test_ratio_on_the_workload_matrices():
    """On a Student-t matrix the variant stores less than the Huffman format
    (about 0.07 bits of headers per value against the Huffman code's
    redundancy), and it stays above the entropy bound."""
    x = workloads.matrix(1, 0).reshape(-1)
    r = oracle.rans_encode(x)
    d = oracle.encode(x, cap=12)
    e, _ = oracle.split(x)
    h = oracle.histogram(e)
    p = h[h > 0] / x.size
    entropy_bytes = x.size + x.size * float(-(p * np.log2(p)).sum()) / 8
    assert entropy_bytes < oracle.rans_stored_bytes(r) < oracle.stored_bytes(d)
