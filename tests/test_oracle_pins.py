"""Pins for the CPU oracle: each test checks it against something other than
itself -- closed forms, hand-derived worked examples, textbook identities,
brute force on tiny alphabets, and invariants the DFloat11 page fixes
("DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70% kích
thước", vi.news.hada.io/topic?id=20542).  No GPU is needed."""
import heapq
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def hist_from(counts, first=0):
    h = np.zeros(256, np.uint64)
    for i, c in enumerate(counts):
        h[first + i] = c
    return h


def cost(h, ln):
    return int(sum(int(h[s]) * int(ln[s]) for s in range(256)))


def kraft(ln):
    return sum(Fraction(1, 2 ** int(l)) for l in ln if l > 0)


def textbook_huffman_cost(counts):
    """Cost of any optimal prefix code = sum of the weights of all merged
    nodes of a Huffman run (a classical identity; independent of ties)."""
    q = [int(c) for c in counts if c > 0]
    if len(q) <= 1:
        return sum(q)  # one symbol gets a 1-bit code
    heapq.heapify(q)
    total = 0
    while len(q) > 1:
        a = heapq.heappop(q)
        b = heapq.heappop(q)
        total += a + b
        heapq.heappush(q, a + b)
    return total


def brute_force_min_cost(counts, max_len):
    """Min sum c*l over every length multiset with Kraft sum <= 1 and
    1 <= l <= max_len (shortest lengths to the largest counts)."""
    cs = sorted((int(c) for c in counts if c > 0), reverse=True)
    m = len(cs)
    best = None
    for lens in itertools.combinations_with_replacement(range(1, max_len + 1), m):
        if sum(Fraction(1, 2 ** l) for l in lens) > 1:
            continue
        c = sum(a * b for a, b in zip(cs, lens))
        best = c if best is None else min(best, c)
    return best


# ------------------------------------------------------------------ split


def test_split_layout_and_inverse_on_every_pattern(olib):
    """[Exponent] 1 sign, 8 exponent, 7 mantissa bits; sign+mantissa byte has
    the sign in bit 7 (reading R1).  merge(split(x)) == x for all 65,536."""
    x = workloads.all_patterns()
    e, sm = oracle.split(x, olib)
    i = np.arange(65536, dtype=np.uint32)
    assert np.array_equal(e, ((i >> 7) & 0xFF).astype(np.uint8))
    assert np.array_equal(sm, (((i >> 8) & 0x80) | (i & 0x7F)).astype(np.uint8))
    # special values keep their fields: +-0, +-inf, a NaN, a subnormal
    for word, expo in [(0x0000, 0), (0x8000, 0), (0x7F80, 255), (0xFF80, 255), (0x7FC1, 255),
                       (0x0001, 0), (0x3F80, 127)]:
        assert e[word] == expo
    assert np.array_equal(oracle.merge(e, sm, olib), x)


def test_histogram_matches_bincount(olib):
    g = np.random.default_rng(0)
    e = g.integers(0, 256, 100_003).astype(np.uint8)
    e[:500] = 7
    assert np.array_equal(oracle.histogram(e, olib),
                          np.bincount(e, minlength=256).astype(np.uint64))
    assert oracle.histogram(np.zeros(0, np.uint8), olib).sum() == 0


def test_entropy_closed_forms(olib):
    assert oracle.entropy(np.ones(256, np.uint64), olib) == pytest.approx(8.0, abs=1e-12)
    assert oracle.entropy(hist_from([5, 5]), olib) == pytest.approx(1.0, abs=1e-12)
    assert oracle.entropy(hist_from([4, 2, 1, 1]), olib) == pytest.approx(1.75, abs=1e-12)
    assert oracle.entropy(hist_from([9]), olib) == 0.0


# ---------------------------------------------------------------- Huffman


@pytest.mark.parametrize("seed", range(40))
def test_huffman_cost_equals_textbook_identity(olib, seed):
    g = np.random.default_rng(seed)
    m = int(g.integers(2, 257))
    h = np.zeros(256, np.uint64)
    syms = g.choice(256, m, replace=False)
    scale = [10, 1000, 1 << 20, 1 << 40][seed % 4]
    h[syms] = g.integers(1, scale, m).astype(np.uint64)
    ln = oracle.huffman_lengths(h, olib)
    assert cost(h, ln) == textbook_huffman_cost(h)
    assert kraft(ln) == 1
    assert all((ln[s] > 0) == (h[s] > 0) for s in range(256))


@pytest.mark.parametrize("seed", range(30))
def test_huffman_optimal_by_brute_force(olib, seed):
    g = np.random.default_rng(100 + seed)
    m = int(g.integers(2, 8))
    counts = g.integers(1, 50, m)
    h = hist_from(counts, first=int(g.integers(0, 240)))
    ln = oracle.huffman_lengths(h, olib)
    assert cost(h, ln) == brute_force_min_cost(counts, m - 1)


@pytest.mark.parametrize("seed", range(20))
def test_entropy_bound(olib, seed):
    """H <= mean code length < H + 1 for an unconstrained Huffman code."""
    g = np.random.default_rng(200 + seed)
    h = np.zeros(256, np.uint64)
    m = int(g.integers(2, 100))
    h[g.choice(256, m, replace=False)] = g.geometric(0.05, m).astype(np.uint64)
    ln = oracle.huffman_lengths(h, olib)
    total = int(h.sum())
    mean = cost(h, ln) / total
    H = oracle.entropy(h, olib)
    assert H - 1e-12 <= mean < H + 1


@pytest.mark.parametrize("k", range(3, 31))
def test_fibonacci_counts_give_lengths_1_to_k_minus_1(olib, k):
    """Counts F_1..F_k: the code lengths are 1, 2, ..., k-1, k-1 (largest
    count shortest) -- the classical worst case for code length."""
    f = workloads.fibonacci_counts(k)
    h = hist_from(f, first=40)
    ln = oracle.huffman_lengths(h, olib)
    got = [int(ln[40 + i]) for i in range(k)][::-1]  # largest count first
    assert got == list(range(1, k)) + [k - 1]


def test_tie_break_reading_hand_cases(olib):
    """Reading R2 (the page names no tie rule).  Counts {1,1,2,2}: merging the
    two 1s gives an internal node of weight 2; leaves precede equal-weight
    internal nodes, so the two 2-leaves merge next: all lengths 2.  (The
    opposite rule would give 1,2,3,3 -- equally optimal.)"""
    ln = oracle.huffman_lengths(hist_from([1, 1, 2, 2], first=10), olib)
    assert [int(x) for x in ln[10:14]] == [2, 2, 2, 2]
    # one symbol: a 1-bit code (Kraft 1/2); empty: nothing
    ln = oracle.huffman_lengths(hist_from([7], first=3), olib)
    assert int(ln[3]) == 1 and int(ln.sum()) == 1
    assert int(oracle.huffman_lengths(np.zeros(256, np.uint64), olib).sum()) == 0


# ---------------------------------------------------------- package-merge


@pytest.mark.parametrize("seed", range(30))
def test_package_merge_optimal_by_brute_force(olib, seed):
    g = np.random.default_rng(300 + seed)
    m = int(g.integers(2, 9))
    cap = int(g.integers(max(1, math.ceil(math.log2(m))), 6))
    counts = g.integers(1, 200, m) ** int(g.integers(1, 3))
    h = hist_from(counts, first=int(g.integers(0, 240)))
    ln = oracle.package_merge(h, cap, olib)
    assert int(ln.max()) <= cap
    assert kraft(ln) == 1
    assert cost(h, ln) == brute_force_min_cost(counts, cap)


@pytest.mark.parametrize("seed", range(10))
def test_package_merge_with_loose_cap_matches_huffman_cost(olib, seed):
    g = np.random.default_rng(400 + seed)
    h = np.zeros(256, np.uint64)
    m = int(g.integers(2, 200))
    h[g.choice(256, m, replace=False)] = g.integers(1, 10**6, m).astype(np.uint64)
    assert cost(h, oracle.package_merge(h, 32, olib)) == textbook_huffman_cost(h)


@pytest.mark.parametrize("k", [5, 6, 7, 8])
def test_fibonacci_cap_small_exact(olib, k):
    """Fibonacci counts with cap k-2: the optimum costs exactly one more than
    the unconstrained Huffman code (brute force)."""
    f = workloads.fibonacci_counts(k)
    h = hist_from(f, first=50)
    ln, _ = oracle.codebook(h, k - 2, olib)
    assert int(ln.max()) <= k - 2 and kraft(ln) == 1
    assert cost(h, ln) == brute_force_min_cost(f, k - 2) == textbook_huffman_cost(f) + 1


def test_fibonacci_cap_32_closed_form(olib):
    """34 Fibonacci counts (14,930,351 values): the unconstrained code is 33
    bits long.  Under the 32-bit cap the code has max length 32, Kraft sum 1,
    and cost between the Huffman cost and Huffman + 1 (the code with lengths
    1..30 and four 32s has cost Huffman + 1 and satisfies the cap)."""
    f = workloads.fibonacci_counts(34)
    assert sum(f) == 14_930_351
    h = hist_from(f, first=100)
    assert int(oracle.huffman_lengths(h, olib).max()) == 33
    ln, _ = oracle.codebook(h, 32, olib)
    hc = textbook_huffman_cost(f)
    witness = list(range(1, 31)) + [32] * 4
    assert kraft([l for l in witness]) == 1
    assert sum(a * b for a, b in zip(sorted(f, reverse=True), witness)) == hc + 1
    assert int(ln.max()) == 32 and kraft(ln) == 1
    assert hc <= cost(h, ln) <= hc + 1


def test_cap_too_small_is_rejected(olib):
    with pytest.raises(ValueError):
        oracle.package_merge(hist_from([1] * 9), 3, olib)


# ---------------------------------------------------- normalise, canonical


@pytest.mark.parametrize("seed", range(10))
def test_normalize_sorts_lengths_by_count(olib, seed):
    g = np.random.default_rng(500 + seed)
    h = np.zeros(256, np.uint64)
    m = int(g.integers(2, 60))
    syms = g.choice(256, m, replace=False)
    h[syms] = g.integers(1, 5, m).astype(np.uint64)  # many ties
    ln0 = oracle.huffman_lengths(h, olib)
    ln = oracle.normalize_lengths(h, ln0, olib)
    assert sorted(ln0.tolist()) == sorted(ln.tolist())
    order = sorted(syms.tolist(), key=lambda s: (-int(h[s]), s))
    got = [int(ln[s]) for s in order]
    assert got == sorted(got)


def test_canonical_rfc1951_worked_example(olib):
    gd = json.load(open(os.path.join(GOLDEN, "rfc1951_canonical.json")))
    ln = np.zeros(256, np.uint8)
    for s, l in zip(gd["symbols"], gd["lengths"]):
        ln[s] = l
    code = oracle.canonical_codes(ln, olib)
    for s, l, want in zip(gd["symbols"], gd["lengths"], gd["codes"]):
        assert format(int(code[s]), f"0{l}b") == want


def test_canonical_uniform_closed_form(olib):
    """All 256 exponents equally frequent: every length is 8 and the code of
    symbol s is s itself."""
    ln, code = oracle.codebook(np.full(256, 3, np.uint64), 32, olib)
    assert set(ln.tolist()) == {8}
    assert np.array_equal(code, np.arange(256, dtype=np.uint32))


def test_canonical_codes_are_prefix_free(olib):
    g = np.random.default_rng(9)
    h = np.zeros(256, np.uint64)
    h[g.choice(256, 80, replace=False)] = g.integers(1, 10**5, 80).astype(np.uint64)
    ln, code = oracle.codebook(h, 32, olib)
    words = [format(int(code[s]), f"0{int(ln[s])}b") for s in range(256) if ln[s]]
    for a, b in itertools.permutations(words, 2):
        assert not b.startswith(a)


# ------------------------------------------------------ stream + metadata


def test_worked_example_golden(olib):
    gd = json.load(open(os.path.join(GOLDEN, "worked_tiny.json")))
    w = np.array([int(x, 16) for x in gd["weights_hex"]], np.uint16)
    enc = oracle.encode(w, lib=olib)
    for s, l in gd["lengths"].items():
        assert int(enc.lengths[int(s)]) == l
        assert format(int(enc.codes[int(s)]), f"0{l}b") == gd["codes"][s]
    assert int((enc.lengths > 0).sum()) == len(gd["lengths"])
    bits = gd["bitstring"] + gd["bitstring_repeat"] * gd["bitstring_repeat_times"]
    assert len(bits) == gd["total_bits"] == enc.total_bits
    want = np.packbits(np.array([int(c) for c in bits.ljust(64 * gd["n_chunks"], "0")], np.uint8))
    assert np.array_equal(enc.stream, want)
    assert enc.gaps.tolist() == gd["gaps"]
    assert enc.gaps_packed.tolist() == gd["gaps_packed"]
    assert enc.block_pos.tolist() == gd["block_pos"]
    assert np.array_equal(oracle.decode(enc, lib=olib), w)
    assert np.array_equal(oracle.decode(enc, chunked=True, lib=olib), w)


def test_all_patterns_stream_is_exponent_bytes(olib):
    """Closed form: with the uniform histogram every code is the 8-bit
    exponent itself, so the stream equals the exponent byte sequence, every
    chunk starts on a code (gaps 0) and block b starts at code 2048*b."""
    x = workloads.all_patterns()
    enc = oracle.encode(x, lib=olib)
    e, _ = oracle.split(x, olib)
    assert enc.total_bits == 8 * 65536
    assert np.array_equal(enc.stream, e)
    assert not enc.gaps.any()
    assert enc.block_pos.tolist() == [2048 * b for b in range(33)]
    assert np.array_equal(oracle.decode(enc, lib=olib), x)
    assert np.array_equal(oracle.decode(enc, chunked=True, lib=olib), x)


@pytest.mark.parametrize("n", [1, 63, 64, 65, 16384, 16385, 40000])
def test_single_symbol_closed_form(olib, n):
    """One exponent value: a 1-bit code '0', n zero bits, every chunk starts
    on a code, block b starts at value 16384*b."""
    x = workloads.constant(n, 0xBC00)
    enc = oracle.encode(x, lib=olib)
    assert int((enc.lengths > 0).sum()) == 1 and int(enc.lengths.max()) == 1
    assert enc.total_bits == n and not enc.stream.any()
    C = (n + 63) // 64
    assert enc.stream.size == 8 * C and enc.gaps.size == C and not enc.gaps.any()
    B = (C + 255) // 256
    assert enc.block_pos.tolist() == [min(16384 * b, n) for b in range(B)] + [n]
    assert np.array_equal(oracle.decode(enc, chunked=True, lib=olib), x)


@pytest.mark.parametrize("reps", [10, 333, 2000])
def test_structured_gaps_closed_form(olib, reps):
    """Repeating [A, B, C] (exponents 127, 126, 125) with equal counts: under
    the reading (equal counts -> lower symbol gets the shorter code) C gets
    1 bit and A, B get 2, so code starts are 5k, 5k+2, 5k+4 and gap[c]
    follows from that arithmetic progression."""
    a, b, c = 0x3F80, 0x3F00, 0x3E80  # exponents 127, 126, 125
    x = np.tile(np.array([a, b, c], np.uint16), reps)
    enc = oracle.encode(x, lib=olib)
    # counts all equal -> normalisation gives the 1-bit code to the lowest symbol (125)
    assert int(enc.lengths[125]) == 1 and int(enc.lengths[126]) == 2 and int(enc.lengths[127]) == 2
    per = [2, 2, 1]  # A=127 (2 bits), B=126 (2 bits), C=125 (1 bit)
    starts, p = [], 0
    for _ in range(reps):
        for l in per:
            starts.append(p)
            p += l
    total = p
    assert enc.total_bits == total
    C = (total + 63) // 64
    want = []
    for ch in range(C):
        nxt = [s for s in starts if s >= 64 * ch]
        want.append((nxt[0] if nxt else total) - 64 * ch)
    assert enc.gaps.tolist() == want
    assert np.array_equal(oracle.decode(enc, chunked=True, lib=olib), x)


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 4097, 100_000, 300_001])
def test_round_trip_and_invariants(olib, n):
    x = workloads.random_bf16(n, seed=n + 1)
    enc = oracle.encode(x, lib=olib)
    assert enc.total_bits == cost(enc.hist, enc.lengths)
    C, B = enc.n_chunks, enc.n_blocks
    assert enc.stream.size == 8 * C and enc.gaps_packed.size == (5 * C + 7) // 8
    assert enc.gaps.size == C and int(enc.gaps.max(initial=0)) <= 31
    pos = enc.block_pos.astype(np.int64)
    assert pos[0] == 0 and pos[-1] == n and np.all(np.diff(pos) >= 0)
    assert np.array_equal(oracle.unpack_gaps(enc.gaps_packed, C, olib), enc.gaps)
    assert np.array_equal(oracle.decode(enc, lib=olib), x)
    assert np.array_equal(oracle.decode(enc, chunked=True, lib=olib), x)
    if int((enc.hist > 0).sum()) >= 2:  # one symbol: 1 bit against H = 0
        H = oracle.entropy(enc.hist, olib)
        assert H - 1e-12 <= enc.total_bits / n < H + 1


def test_every_pattern_shuffled_round_trip(olib):
    x = workloads.shuffled_patterns(4)
    enc = oracle.encode(x, lib=olib)
    assert np.array_equal(oracle.decode(enc, chunked=True, lib=olib), x)


def test_fibonacci_cap_stream_round_trip(olib):
    x = workloads.fibonacci_exponents(34)
    enc = oracle.encode(x, lib=olib)
    assert int(enc.lengths.max()) == 32
    assert int(enc.gaps.max()) <= 31
    assert np.array_equal(oracle.decode(enc, chunked=True, lib=olib), x)


def test_corrupt_metadata_is_detected(olib):
    x = workloads.random_bf16(50_000, seed=3)
    enc = oracle.encode(x, lib=olib)
    bad = enc.block_pos.copy()
    bad[1] += 1
    with pytest.raises(ValueError):
        oracle.decode_chunked_exponents(enc.stream, enc.gaps, bad, enc.total_bits, enc.n,
                                        enc.lengths, enc.codes, olib)
    g = enc.gaps.copy()
    g[3] = (g[3] + 1) % 32
    with pytest.raises(ValueError):
        oracle.decode_chunked_exponents(enc.stream, g, enc.block_pos, enc.total_bits, enc.n,
                                        enc.lengths, enc.codes, olib)


def test_workload1_statistics_band(olib):
    """Sanity band from the page ([Exponent]: exponent entropy about 2.6 bits,
    about 40 of 256 values used; [Format]: about 11 bits per weight).  The
    synthetic Gaussian stand-in lands close to these figures."""
    x = workloads.matrix(1, 0)
    enc = oracle.encode(x, lib=olib)
    H = oracle.entropy(enc.hist, olib)
    assert 2.3 < H < 2.9
    assert 10 <= int((enc.hist > 0).sum()) <= 60
    bits_per_weight = 8 + enc.total_bits / enc.n
    assert 10.3 < bits_per_weight < 11.2


# --------------------------------------------------------------- run index (R12)
# For run r of block b (its chunks 2r and 2r+1), the number of codes that start
# in the block before the run.  [Kernel] fixes one output position per thread
# block; this is the same count for each pair of chunks of a block.


def _run_index_by_search(x, enc):
    """The same quantity by a different route: code starts from the cumulative
    sum of the code lengths, counted per boundary with a binary search."""
    e, _ = oracle.split(x)
    lens = enc.lengths[e].astype(np.uint64)
    starts = np.cumsum(lens) - lens
    runs = enc.n_blocks * 128
    bounds = np.arange(runs, dtype=np.uint64) * 128
    block_bounds = (np.arange(runs, dtype=np.uint64) // 128) * 16384
    return (np.searchsorted(starts, bounds, side="left")
            - np.searchsorted(starts, block_bounds, side="left")).astype(np.uint16)


def test_run_index_all_patterns_closed_form(olib):
    """8-bit codes: 16 codes start in every 128-bit run, so run r of any
    block starts at output 16 r within it."""
    x = workloads.all_patterns()
    enc = oracle.encode(x)
    ri = oracle.run_index(x, enc.lengths, enc.total_bits)
    assert ri.size == 32 * 128
    assert np.array_equal(ri, np.tile(np.arange(128, dtype=np.uint16) * 16, 32))


@pytest.mark.parametrize("n", [1, 128, 129, 16384, 16385, 40000])
def test_run_index_single_symbol_closed_form(olib, n):
    """One value with a 1-bit code: 128 codes per run, and runs past the end
    of the stream hold their block's total."""
    x = workloads.constant(n, 0xBC00)
    enc = oracle.encode(x)
    ri = oracle.run_index(x, enc.lengths, enc.total_bits).astype(np.int64)
    b, r = np.divmod(np.arange(ri.size), 128)
    in_block = np.minimum(n - 16384 * b, 16384)
    assert np.array_equal(ri, np.minimum(128 * r, in_block))


def test_run_index_hand_example(olib):
    """64 values of a 1-bit code, then 40 of a 2-bit code: bits 0..63 hold 64
    codes, the 2-bit codes start at 64, 66, ..., 142.  The run boundary at
    bit 128 has 64 + 32 code starts before it; every later run of the block
    (past the end of the 144-bit stream) holds the block total, 104."""
    lengths = np.zeros(256, np.uint8)
    codes = np.zeros(256, np.uint32)
    lengths[10], codes[10] = 1, 0b0
    lengths[20], codes[20] = 2, 0b10
    x = np.array([10 << 7] * 64 + [20 << 7] * 40, np.uint16)
    enc = oracle.encode(x, lengths=lengths, codes=codes)
    assert enc.total_bits == 144
    ri = oracle.run_index(x, lengths, 144)
    assert ri.tolist() == [0, 96] + [104] * 126


@pytest.mark.parametrize("n", [7, 4097, 100_000, 300_001])
def test_run_index_matches_binary_search_and_block_positions(olib, n):
    x = workloads.random_bf16(n, seed=31 + n)
    enc = oracle.encode(x, cap=11)
    ri = oracle.run_index(x, enc.lengths, enc.total_bits)
    assert np.array_equal(ri, _run_index_by_search(x, enc))
    per_block = ri.reshape(-1, 128).astype(np.int64)
    totals = np.diff(enc.block_pos.astype(np.int64))
    assert (per_block[:, 0] == 0).all()
    assert (np.diff(per_block, axis=1) >= 0).all()
    assert (per_block[:, -1] <= totals).all()


# ----------------------------------------------------------- segment index (R13)
# For every 64th value, the stream bit at which its code starts; then
# total_bits.  The converse of the block positions: output -> stream bit.


def _code_at(stream, bit, length):
    """The length bits of the stream starting at bit, MSB first (R5), read
    bit by bit from the bytes."""
    v = 0
    for k in range(bit, bit + length):
        v = (v << 1) | ((int(stream[k >> 3]) >> (7 - (k & 7))) & 1)
    return v


def test_segment_index_all_patterns_closed_form(olib):
    """8-bit codes: value 64j starts at bit 512j; 1024 segments, then 2^19."""
    x = workloads.all_patterns()
    enc = oracle.encode(x)
    seg = oracle.segment_index(x, enc.lengths, enc.total_bits)
    assert np.array_equal(seg, 512 * np.arange(1025, dtype=np.uint32))


@pytest.mark.parametrize("n", [1, 63, 64, 65, 4096, 40001])
def test_segment_index_single_symbol_closed_form(olib, n):
    """One value with a 1-bit code: value 64j starts at bit 64j; the last
    entry is n (= total_bits)."""
    x = workloads.constant(n, 0xBC00)
    enc = oracle.encode(x)
    seg = oracle.segment_index(x, enc.lengths, enc.total_bits).astype(np.int64)
    S = (n + 63) // 64
    assert seg.size == S + 1
    assert np.array_equal(seg[:S], 64 * np.arange(S)) and seg[S] == n


def test_segment_index_hand_example(olib):
    """64 values of a 1-bit code, then 40 of a 2-bit code (144 bits): value
    0 starts at bit 0, value 64 (the first 2-bit code) at bit 64."""
    lengths = np.zeros(256, np.uint8)
    codes = np.zeros(256, np.uint32)
    lengths[10], codes[10] = 1, 0b0
    lengths[20], codes[20] = 2, 0b10
    x = np.array([10 << 7] * 64 + [20 << 7] * 40, np.uint16)
    enc = oracle.encode(x, lengths=lengths, codes=codes)
    assert oracle.segment_index(x, lengths, 144).tolist() == [0, 64, 144]
    assert oracle.segment_index(x[:64], lengths, 64).tolist() == [0, 64]


@pytest.mark.parametrize("n,cap", [(7, 11), (4097, 11), (100_000, 11), (300_001, 11), (70_001, 32)])
def test_segment_index_against_stream_and_block_positions(olib, n, cap):
    """Against the encoder's own arrays: the stream holds value 64j's code at
    bit seg[j]; segments use between 64 x the shortest and 64 x the longest
    code; and the segment starts before block b's first bit are exactly the
    multiples of 64 below block_pos[b] (the codes that start before it)."""
    x = workloads.random_bf16(n, seed=77 + n) if cap == 11 else workloads.fibonacci_exponents(26)[:n]
    enc = oracle.encode(x, cap=cap)
    seg = oracle.segment_index(x, enc.lengths, enc.total_bits).astype(np.int64)
    e, _ = oracle.split(x)
    S = (n + 63) // 64
    assert seg.size == S + 1 and seg[0] == 0 and seg[S] == enc.total_bits
    for j in range(0, S, max(1, S // 200)):
        v = int(e[64 * j])
        L = int(enc.lengths[v])
        assert _code_at(enc.stream, int(seg[j]), L) == int(enc.codes[v]), j
    used = enc.lengths[enc.lengths > 0]
    d = np.diff(seg)
    full = np.minimum(64, n - 64 * np.arange(S))
    assert (d >= full * int(used.min())).all() and (d <= full * int(used.max())).all()
    for b in range(enc.block_pos.size):
        below = int((seg[:S] < 16384 * b).sum())
        assert below == (int(enc.block_pos[b]) + 63) // 64, b
