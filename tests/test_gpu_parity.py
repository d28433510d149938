"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, bit for
bit -- histogram, every encoded array (stream, gaps, block positions,
sign/mantissa plane) and the decoded BF16 words -- on edge cases and on all
five workloads at full size, in the launch configuration bench.py times.

Expected values come from the oracle only.  Where the expected decode output
is the input itself, that is the oracle's own result: its round trip is the
identity (pinned in test_oracle_pins.py) and small cases call it explicitly.

Every case runs under three code-length caps: 11 (the codec default, the
decode table's reach: the fast path), 12 (codes one bit longer than the
table: the length search for the rarest values) and 32 (the format's limit).
The oracle builds its codebook with the same cap."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def codec():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    import lossless_bf16_weight_df11_b200.codec as c
    return c


def to_dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x).reshape(-1).view(np.int16)).cuda()


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)


def assert_encoded_equal(m, enc):
    h = m.host_arrays()
    assert m.total_bits == enc.total_bits
    assert np.array_equal(h["lengths"], enc.lengths)
    assert np.array_equal(h["stream"], enc.stream), "stream differs"
    assert np.array_equal(h["gaps"], enc.gaps_packed), "gaps differ"
    assert np.array_equal(h["block_pos"], enc.block_pos), "block positions differ"
    assert np.array_equal(h["sign_mantissa"], enc.sign_mantissa), "sign/mantissa differ"


CAPS = [11, 12, 32]

# the three decoders: with the run index (the default when a matrix has one),
# with the segment index alone, and with neither (per-unit prefix sums)
DECODERS = {"run": {}, "segment": {"run_index": False},
            "plain": {"run_index": False, "seg_index": False}}


def assert_run_index_equal(m, x, enc):
    if enc.n == 0:
        assert m.run_index is None
        return
    want = oracle.run_index(x, enc.lengths, enc.total_bits)
    got = m.run_index[: want.size].cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want), "run index differs"


def assert_seg_index_equal(m, x, enc):
    if enc.n == 0:
        assert m.seg_index is None
        return
    want = oracle.segment_index(x, enc.lengths, enc.total_bits)
    got = m.seg_index[: want.size].cpu().numpy().view(np.uint32)
    assert np.array_equal(got, want), "segment index differs"


def full_check(codec, x: np.ndarray, cap: int, call_oracle_decode: bool = True):
    x = np.ascontiguousarray(x, np.uint16).reshape(-1)
    enc = oracle.encode(x, cap=cap)
    w = to_dev(x)
    hist = codec.histogram(w).cpu().numpy().view(np.uint64)
    assert np.array_equal(hist, enc.hist), "histogram differs"
    m = codec.compress(w, cap=cap)
    assert_encoded_equal(m, enc)
    assert_run_index_equal(m, x, enc)
    assert_seg_index_equal(m, x, enc)
    expected = oracle.decode(enc, chunked=True) if call_oracle_decode else x
    for name, kw in DECODERS.items():
        out = codec.decompress(m, **kw)
        assert np.array_equal(bits_of(out), expected), f"decode ({name}) of GPU-encoded data differs"
    # decode of the oracle's own buffers (independent of the GPU encoder)
    cb = codec.codebook_from_lengths(enc.lengths, enc.codes)
    mo = codec.from_host_arrays(x.shape, enc.n, enc.total_bits, cb, enc.stream, enc.gaps_packed,
                                enc.block_pos, enc.sign_mantissa, w.device)
    assert_run_index_equal(mo, x, enc)
    assert_seg_index_equal(mo, x, enc)
    out2 = codec.decompress(mo)
    assert np.array_equal(bits_of(out2), expected), "decode of oracle-encoded data differs"
    return m, enc


@pytest.mark.parametrize("cap", CAPS)
@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 15, 16, 17, 4097, 65_537, 1_000_003])
def test_sizes_and_ragged_tails(codec, n, cap):
    full_check(codec, workloads.random_bf16(n, seed=1000 + n), cap)


@pytest.mark.parametrize("cap", CAPS)
def test_every_bit_pattern(codec, cap):
    m, enc = full_check(codec, workloads.all_patterns(), cap)
    assert np.array_equal(m.host_arrays()["stream"], oracle.split(workloads.all_patterns())[0])


@pytest.mark.parametrize("cap", CAPS)
def test_every_bit_pattern_shuffled(codec, cap):
    full_check(codec, workloads.shuffled_patterns(4), cap)


@pytest.mark.parametrize("cap", CAPS)
@pytest.mark.parametrize("n", [1, 64, 65, 16_384, 16_385, 1_000_000])
def test_single_symbol(codec, n, cap):
    full_check(codec, workloads.constant(n, 0xBC00), cap)


@pytest.mark.parametrize("cap", CAPS)
def test_two_symbols_and_all_equal_words(codec, cap):
    g = np.random.default_rng(3)
    x = np.where(g.random(300_000) < 0.7, 0x3F80, 0xC000).astype(np.uint16)
    full_check(codec, x, cap)
    full_check(codec, workloads.constant(123_457, 0x0000), cap)


@pytest.mark.parametrize("cap", CAPS)
def test_worked_example(codec, cap):
    import json, os
    gd = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_tiny.json")))
    x = np.array([int(v, 16) for v in gd["weights_hex"]], np.uint16)
    m, _ = full_check(codec, x, cap)
    h = m.host_arrays()
    assert h["gaps"].tolist() == gd["gaps_packed"] and h["block_pos"].tolist() == gd["block_pos"]


def test_fibonacci_length_cap(codec):
    """14,930,351 values whose exponent counts are Fibonacci numbers: the code
    needs the 32-bit cap, so 21 of the codes are longer than the 11-bit
    decode table and take the length-search path."""
    m, enc = full_check(codec, workloads.fibonacci_exponents(34), 32, call_oracle_decode=False)
    assert int(enc.lengths.max()) == 32


@pytest.mark.parametrize("cap", [11, 12])
def test_fibonacci_at_table_cap(codec, cap):
    """The same input under the table's 11-bit cap (package-merge shortens
    every code to the table's reach) and one bit above it."""
    m, enc = full_check(codec, workloads.fibonacci_exponents(34), cap, call_oracle_decode=False)
    assert int(enc.lengths.max()) == cap


@pytest.mark.parametrize("cap", CAPS)
@pytest.mark.parametrize("wid", [1, 2, 4])
def test_workload_single_matrix(codec, wid, cap):
    x = workloads.matrix(wid, 0)
    m, enc = full_check(codec, x, cap, call_oracle_decode=(wid == 1))
    assert m.stored_bytes == oracle.stored_bytes(enc)


@pytest.mark.parametrize("wid,cap", [(3, 11), (3, 32), (5, 11), (5, 12), (5, 32)])
def test_workload_block_batched(codec, wid, cap):
    """A whole transformer block: per-matrix codebooks, one decode launch
    (the bench configuration, cap 11; and caps 12 and 32)."""
    names = [nm for nm, _ in workloads.WORKLOADS[wid][1]]
    mats, xs = [], []
    for i, _ in enumerate(names):
        x = workloads.matrix(wid, i).reshape(-1)
        enc = oracle.encode(x, cap=cap)
        m = codec.compress(to_dev(x), cap=cap)
        assert_encoded_equal(m, enc)
        assert_run_index_equal(m, x, enc)
        assert_seg_index_equal(m, x, enc)
        mats.append(m)
        xs.append(x)
        del enc
    for name, kw in DECODERS.items():
        outs = codec.decompress_block(mats, **kw)
        for x, o in zip(xs, outs):
            assert np.array_equal(bits_of(o), x), name
        del outs


@pytest.mark.parametrize("use_index", [True, False])
@pytest.mark.parametrize("cap", CAPS)
def test_decode_reports_corrupt_positions_without_fault(codec, cap, use_index):
    """Block positions are read by the run-index and plain decoders (the
    segment decoder does not read them)."""
    x = workloads.random_bf16(2_000_000, seed=9)
    m = codec.compress(to_dev(x), cap=cap)
    pos = m.block_pos.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b in (3, 4):  # a position inside a decode unit and one between two units
        m.block_pos[b] += 5
        status.zero_()
        codec.decompress(m, status=status, run_index=use_index, seg_index=False)
        assert int(status.item()) == 4  # DF11_ERR_CORRUPT
        m.block_pos.copy_(pos)
    m.block_pos[5] = int(m.n) + 100  # beyond the matrix: must not be dereferenced
    status.zero_()
    codec.decompress(m, status=status, run_index=use_index, seg_index=False)
    assert int(status.item()) == 4
    m.block_pos.copy_(pos)
    m.stream[1000:1010] ^= 0x5A  # flipped stream bits change the counts
    status.zero_()
    out = codec.decompress(m, status=status, run_index=use_index, seg_index=False)
    torch.cuda.synchronize()
    assert int(status.item()) in (0, 4)
    m.stream[1000:1010] ^= 0x5A
    status.zero_()
    out = codec.decompress(m, status=status, run_index=use_index, seg_index=False)
    assert int(status.item()) == 0 and np.array_equal(bits_of(out), x)


def test_decode_reports_corrupt_run_index_without_fault(codec):
    """Run-index entries that disagree with the stream, or point past their
    block, are reported as corrupt; the decode of the intact index after
    them is exact (rejected units leave nothing behind)."""
    x = workloads.random_bf16(2_000_000, seed=10)
    m = codec.compress(to_dev(x))
    ri = m.run_index.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for k, v in ((5, 1), (128, 3), (300, -7), (129, 30000), (255, 32767)):
        m.run_index[k] += v
        status.zero_()
        codec.decompress(m, status=status)
        assert int(status.item()) == 4, (k, v)
        m.run_index.copy_(ri)
    status.zero_()
    out = codec.decompress(m, status=status)
    assert int(status.item()) == 0 and np.array_equal(bits_of(out), x)


@pytest.mark.parametrize("cap", CAPS)
def test_decode_reports_corrupt_segment_index_without_fault(codec, cap):
    """Segment-index entries that disagree with the stream (one bit off, far
    off, past the stream, out of order) are reported as corrupt: the decode
    of a segment must end exactly where the next one starts.  Stream bits
    flipped under an intact index are reported or decode silently (the
    format has no checksum), never fault; the decode of intact data after
    them is exact."""
    x = workloads.random_bf16(2_000_000, seed=11)
    m = codec.compress(to_dev(x), cap=cap)
    si = m.seg_index.clone()
    S = (m.n + 63) // 64
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for k, v in ((5, 1), (31, -1), (32, 9), (1000, 100_000), (S - 1, 3), (S, 7),
                 (700, 1 << 31), (701, -(1 << 20))):
        m.seg_index[k] = int(si[k]) + v if 0 <= int(si[k]) + v < (1 << 31) else (1 << 31) - 1
        status.zero_()
        codec.decompress(m, status=status, run_index=False)
        assert int(status.item()) == 4, (k, v)
        m.seg_index.copy_(si)
    m.stream[5000:5010] ^= 0x5A
    status.zero_()
    codec.decompress(m, status=status, run_index=False)
    torch.cuda.synchronize()
    assert int(status.item()) in (0, 4)
    m.stream[5000:5010] ^= 0x5A
    status.zero_()
    out = codec.decompress(m, status=status, run_index=False)
    assert int(status.item()) == 0 and np.array_equal(bits_of(out), x)


def test_encode_reports_value_without_code(codec):
    import lossless_bf16_weight_df11_b200 as df11
    x = workloads.random_bf16(100_000, seed=4)
    st, cb = df11.df11_build_codebook(oracle.histogram(oracle.split(x[:50_000])[0]), 32)
    missing = [s for s in range(256) if cb.len[s] == 0]
    x[77] = (missing[0] << 7) | 1
    with pytest.raises(df11.DF11Error):
        codec.compress(to_dev(x), codebook=cb)


def test_compress_block_matches_compress(codec):
    """The batched compressor (two host round trips for all matrices) gives,
    array for array, what compress() gives matrix by matrix: the Llama-3-8B
    block and a list of edge cases (empty, one value, a ragged tail, one
    symbol)."""
    import lossless_bf16_weight_df11_b200 as df11
    cases = [[workloads.matrix(3, i) for i in range(len(workloads.WORKLOADS[3][1]))],
             [workloads.random_bf16(0, seed=1), workloads.random_bf16(1, seed=2),
              workloads.random_bf16(1_000_003, seed=3), workloads.constant(65_537, 0x3F80),
              workloads.fibonacci_exponents(34)]]
    for xs in cases:
        ws = [to_dev(x) for x in xs]
        got = codec.compress_block(ws)
        for w, g in zip(ws, got):
            m = codec.compress(w)
            a, b = m.host_arrays(), g.host_arrays()
            for key in ("lengths", "stream", "gaps", "block_pos", "sign_mantissa"):
                assert np.array_equal(a[key], b[key]), key
            assert m.total_bits == g.total_bits and m.max_block_codes == g.max_block_codes
            assert torch.equal(m.tables, g.tables)
        outs = codec.decompress_block([g for g in got if g.n])
        for x, o in zip([x for x in xs if x.size], outs):
            assert np.array_equal(bits_of(o), np.ascontiguousarray(x).reshape(-1))
        del got


def test_batch_larger_than_one_launch(codec):
    """More matrices than one launch takes (DF11_MAX_BATCH = 32): the call
    splits them; every output must still be exact (sizes vary, one is empty,
    one has 1-bit codes)."""
    xs = [workloads.random_bf16(1_000 + 37_000 * i, seed=500 + i) for i in range(38)]
    xs[5] = workloads.random_bf16(0, seed=1)
    xs[17] = workloads.constant(70_001, 0x3F80)
    mats = codec.compress_block([to_dev(x) for x in xs])
    outs = codec.decompress_block([m for m in mats if m.n])
    for x, o in zip([x for x in xs if x.size], outs):
        assert np.array_equal(bits_of(o), x)
