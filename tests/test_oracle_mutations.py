"""Do the oracle's pins catch plausible mistakes?  Each case plants one mistake
in a temporary copy of the oracle's C source (on the CPU; the real source is
untouched), builds it, and checks that at least one pin fails on it, while the
unmodified oracle passes them all."""
import json
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
import workloads
import test_oracle_rans as rp
from test_oracle_pins import GOLDEN, _run_index_by_search, cost, kraft, textbook_huffman_cost, hist_from

MUTATIONS = {
    "lsb_first_bits": [("(uint8_t)(0x80u >> (k & 7u))", "(uint8_t)(0x01u << (k & 7u))"),
                       ("(7u - (unsigned)(k & 7u))", "((unsigned)(k & 7u))")],
    "internal_node_first_on_ties": [("if (best < 0 || weight[id] < weight[best]) best = id;",
                                     "if (best < 0 || weight[id] <= weight[best]) best = id;")],
    "huffman_depth_off_by_one": [("    int depth = 0;\n", "    int depth = 1;\n")],
    "package_merge_takes_one_more": [("size_t take = (size_t)2 * (size_t)(m - 1);",
                                      "size_t take = (size_t)2 * (size_t)m - 1;")],
    "canonical_codes_descending": [("  for (int s = 0; s < 256; s++) {\n    code[s] = 0;",
                                    "  for (int s = 255; s >= 0; s--) {\n    code[s] = 0;")],
    "normalise_longest_to_frequent": [("int swap = hist[a] < hist[b] || (hist[a] == hist[b] && a > b);",
                                       "int swap = hist[a] > hist[b] || (hist[a] == hist[b] && a > b);")],
    "gap_off_by_one": [("gap[next_chunk] = (uint8_t)(start - next_chunk * OR_CHUNK_BITS);",
                        "gap[next_chunk] = (uint8_t)(start - next_chunk * OR_CHUNK_BITS + 1);")],
    "block_pos_counts_inclusive": [("pos[next_block] = (uint32_t)i;",
                                    "pos[next_block] = (uint32_t)(i + 1);")],
    "run_index_counts_boundary_code": [("    while (next_run < runs && next_run * run_bits <= bit) {",
                                        "    while (next_run < runs && next_run * run_bits < bit) {")],
    "run_index_not_reset_per_block": [("      if (next_run % runs_per_block == 0) block_first = i;\n",
                                       "      if (next_run == 0) block_first = i;\n")],
    "segment_index_after_the_code": [("    if (i % 64 == 0) seg[i / 64] = (uint32_t)bit; /* code i starts here */\n    bit += l;",
                                      "    bit += l;\n    if (i % 64 == 0) seg[i / 64] = (uint32_t)bit; /* code i starts here */")],
    "segment_index_one_value_early": [("    if (i % 64 == 0) seg[i / 64] = (uint32_t)bit;",
                                       "    if (i % 64 == 63) seg[i / 64] = (uint32_t)bit;")],
    "segment_index_ends_with_n": [("  seg[segments] = (uint32_t)total_bits;", "  seg[segments] = (uint32_t)n;")],
    "sign_in_bit_0": [("sign_mantissa[i] = (uint8_t)((sign << 7) | mant); /* R1 */",
                       "sign_mantissa[i] = (uint8_t)((mant << 1) | sign); /* R1 */"),
                      ("unsigned sign = (sign_mantissa[i] >> 7) & 1u;\n    unsigned mant = sign_mantissa[i] & 0x7Fu;",
                       "unsigned sign = sign_mantissa[i] & 1u;\n    unsigned mant = sign_mantissa[i] >> 1;")],
    "tail_chunk_not_clipped": [("      if (limit > total_bits) limit = total_bits;\n      if (gap[c] > 31)",
                                "      if (gap[c] > 31)")],
    "canonical_no_shift": [("    c = (c + bl_count[bits - 1]) << 1;", "    c = (c + bl_count[bits - 1]);")],
    "rans_renorm_strict": [("if ((uint64_t)x[l] >= ((uint64_t)f << 20)) {",
                            "if ((uint64_t)x[l] > ((uint64_t)f << 20)) {")],
    "rans_threshold_one_bit_low": [("if ((uint64_t)x[l] >= ((uint64_t)f << 20)) {",
                                    "if ((uint64_t)x[l] >= ((uint64_t)f << 19)) {")],
    "rans_words_in_emission_order": [("uint16_t wv = words[nw - 1 - j];", "uint16_t wv = words[j];")],
    "rans_cum_starts_at_one": [("  cum[0] = 0;\n  for (int s = 0; s < 256; s++) cum[s + 1]",
                                "  cum[0] = 1;\n  for (int s = 0; s < 256; s++) cum[s + 1]")],
    "rans_ties_to_larger_symbol": [("if (pick < 0 || d > best) { pick = s; best = d; }",
                                    "if (pick < 0 || d >= best) { pick = s; best = d; }")],
    "rans_initial_state_off": [("for (unsigned l = 0; l < OR_RANS_LANES; l++) x[l] = OR_RANS_L;",
                                "for (unsigned l = 0; l < OR_RANS_LANES; l++) x[l] = OR_RANS_L + 16;")],
    "rans_segment_start_inclusive": [("      first += seg_words[g];\n    }",
                                      "    }")],
    "rans_lanes_forward_in_encoder": [("for (int l = (int)OR_RANS_LANES - 1; l >= 0; l--) {",
                                       "for (int l = 0; l < (int)OR_RANS_LANES; l++) {")],
}


def _check_uniform(lib):
    x = workloads.all_patterns()
    enc = oracle.encode(x, lib=lib)
    e, _ = oracle.split(x, lib)
    assert np.array_equal(enc.stream, e)
    assert np.array_equal(enc.codes, np.arange(256, dtype=np.uint32))
    assert enc.block_pos.tolist() == [2048 * b for b in range(33)]


def _check_tie(lib):
    ln = oracle.huffman_lengths(hist_from([1, 1, 2, 2], first=10), lib)
    assert [int(v) for v in ln[10:14]] == [2, 2, 2, 2]


def _check_costs(lib):
    g = np.random.default_rng(5)
    for _ in range(5):
        h = np.zeros(256, np.uint64)
        m = int(g.integers(3, 120))
        h[g.choice(256, m, replace=False)] = g.integers(1, 10**5, m).astype(np.uint64)
        ln, _ = oracle.codebook(h, 32, lib)
        assert kraft(ln) == 1 and cost(h, ln) == textbook_huffman_cost(h)
        assert kraft(oracle.huffman_lengths(h, lib)) == 1
    f = workloads.fibonacci_counts(7)
    ln, _ = oracle.codebook(hist_from(f, first=50), 5, lib)
    assert kraft(ln) == 1 and cost(hist_from(f, first=50), ln) == textbook_huffman_cost(f) + 1


def _check_golden(lib):
    gd = json.load(open(os.path.join(GOLDEN, "worked_tiny.json")))
    w = np.array([int(x, 16) for x in gd["weights_hex"]], np.uint16)
    enc = oracle.encode(w, lib=lib)
    bits = gd["bitstring"] + gd["bitstring_repeat"] * gd["bitstring_repeat_times"]
    want = np.packbits(np.array([int(c) for c in bits.ljust(128, "0")], np.uint8))
    assert np.array_equal(enc.stream, want)
    assert enc.gaps.tolist() == gd["gaps"] and enc.block_pos.tolist() == gd["block_pos"]
    assert enc.gaps_packed.tolist() == gd["gaps_packed"]


def _check_layout(lib):
    x = workloads.all_patterns()
    _, sm = oracle.split(x, lib)
    i = np.arange(65536, dtype=np.uint32)
    assert np.array_equal(sm, (((i >> 8) & 0x80) | (i & 0x7F)).astype(np.uint8))


def _check_round_trip(lib):
    for n in (9, 4097, 70_001):
        x = workloads.random_bf16(n, seed=n)
        enc = oracle.encode(x, lib=lib)
        assert np.array_equal(oracle.decode(enc, lib=lib), x)
        assert np.array_equal(oracle.decode(enc, chunked=True, lib=lib), x)


def _check_run_index(lib):
    x = workloads.all_patterns()
    enc = oracle.encode(x, lib=lib)
    ri = oracle.run_index(x, enc.lengths, enc.total_bits, lib)
    assert np.array_equal(ri, np.tile(np.arange(128, dtype=np.uint16) * 16, 32))
    x = workloads.random_bf16(100_000, seed=3)
    enc = oracle.encode(x, cap=11, lib=lib)
    assert np.array_equal(oracle.run_index(x, enc.lengths, enc.total_bits, lib),
                          _run_index_by_search(x, enc))


def _check_segment_index(lib):
    x = workloads.all_patterns()
    enc = oracle.encode(x, lib=lib)
    assert np.array_equal(oracle.segment_index(x, enc.lengths, enc.total_bits, lib),
                          512 * np.arange(1025, dtype=np.uint32))
    x = workloads.random_bf16(100_003, seed=5)
    enc = oracle.encode(x, cap=11, lib=lib)
    seg = oracle.segment_index(x, enc.lengths, enc.total_bits, lib).astype(np.int64)
    assert seg[-1] == enc.total_bits
    for b in range(enc.block_pos.size):
        assert int((seg[:-1] < 16384 * b).sum()) == (int(enc.block_pos[b]) + 63) // 64


def _check_rans(lib):
    f = oracle.rans_freqs(rp.hist_of({0: 1, 1: 1, 2: 1}), lib)
    assert f[:3].tolist() == [1366, 1365, 1365]
    for case in rp.golden_cases():
        w = rp.weights_with_exponents(rp.golden_exponents(case))
        enc = oracle.rans_encode(w, freq=rp.freq_array(case["freq"]), lib=lib)
        assert enc.stream.tobytes() == rp.unit_bytes_from_fields(case)
    x = workloads.shuffled_patterns(copies=1, seed=11)[: 3 * 16384 + 77]
    enc = oracle.rans_encode(x, freq=np.full(256, 16, np.uint32), lib=lib)
    assert np.array_equal(oracle.rans_decode(enc, lib=lib), x)
    for n in (65, 40_000):
        x = workloads.random_bf16(n, seed=n)
        enc = oracle.rans_encode(x, lib=lib)
        assert np.array_equal(oracle.rans_decode(enc, lib=lib), x)


CHECKS = [_check_uniform, _check_tie, _check_costs, _check_golden, _check_layout, _check_round_trip,
          _check_run_index, _check_segment_index, _check_rans]


def _failures(lib):
    bad = []
    for chk in CHECKS:
        try:
            chk(lib)
        except (AssertionError, ValueError):
            bad.append(chk.__name__)
    return bad


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="df11_oracle_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmodified_oracle_passes_every_check(olib):
    assert _failures(olib) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(workdir, name):
    src = open(oracle._SRC).read()
    for old, new in MUTATIONS[name]:
        assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
        src = src.replace(old, new)
    path = os.path.join(workdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src)
    lib = oracle.load(oracle.build(force=True, src=path, out=os.path.join(workdir, f"lib{name}.so")))
    assert _failures(lib), f"no pin caught the planted mistake {name}"
