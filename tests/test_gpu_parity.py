"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, bit for
bit -- histogram, every encoded array (stream, gaps, block positions,
sign/mantissa plane) and the decoded BF16 words -- on edge cases and on all
five workloads at full size, in the launch configuration bench.py times.

Expected values come from the oracle only.  Where the expected decode output
is the input itself, that is the oracle's own result: its round trip is the
identity (pinned in test_oracle_pins.py) and small cases call it explicitly."""
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


def full_check(codec, x: np.ndarray, call_oracle_decode: bool = True):
    x = np.ascontiguousarray(x, np.uint16).reshape(-1)
    enc = oracle.encode(x)
    w = to_dev(x)
    hist = codec.histogram(w).cpu().numpy().view(np.uint64)
    assert np.array_equal(hist, enc.hist), "histogram differs"
    m = codec.compress(w)
    assert_encoded_equal(m, enc)
    expected = oracle.decode(enc, chunked=True) if call_oracle_decode else x
    out = codec.decompress(m)
    assert np.array_equal(bits_of(out), expected), "decode of GPU-encoded data differs"
    # decode of the oracle's own buffers (independent of the GPU encoder)
    cb = codec.codebook_from_lengths(enc.lengths, enc.codes)
    mo = codec.from_host_arrays(x.shape, enc.n, enc.total_bits, cb, enc.stream, enc.gaps_packed,
                                enc.block_pos, enc.sign_mantissa, w.device)
    out2 = codec.decompress(mo)
    assert np.array_equal(bits_of(out2), expected), "decode of oracle-encoded data differs"
    return m, enc


@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 15, 16, 17, 4097, 65_537, 1_000_003])
def test_sizes_and_ragged_tails(codec, n):
    full_check(codec, workloads.random_bf16(n, seed=1000 + n))


def test_every_bit_pattern(codec):
    m, enc = full_check(codec, workloads.all_patterns())
    assert np.array_equal(m.host_arrays()["stream"], oracle.split(workloads.all_patterns())[0])


def test_every_bit_pattern_shuffled(codec):
    full_check(codec, workloads.shuffled_patterns(4))


@pytest.mark.parametrize("n", [1, 64, 65, 16_384, 16_385, 1_000_000])
def test_single_symbol(codec, n):
    full_check(codec, workloads.constant(n, 0xBC00))


def test_two_symbols_and_all_equal_words(codec):
    g = np.random.default_rng(3)
    x = np.where(g.random(300_000) < 0.7, 0x3F80, 0xC000).astype(np.uint16)
    full_check(codec, x)
    full_check(codec, workloads.constant(123_457, 0x0000))


def test_worked_example(codec):
    import json, os
    gd = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_tiny.json")))
    x = np.array([int(v, 16) for v in gd["weights_hex"]], np.uint16)
    m, _ = full_check(codec, x)
    h = m.host_arrays()
    assert h["gaps"].tolist() == gd["gaps_packed"] and h["block_pos"].tolist() == gd["block_pos"]


def test_fibonacci_length_cap(codec):
    """14,930,351 values whose exponent counts are Fibonacci numbers: the code
    needs the 32-bit cap, so 20 of the codes are longer than the 12-bit
    decode table and take the length-search path."""
    m, enc = full_check(codec, workloads.fibonacci_exponents(34), call_oracle_decode=False)
    assert int(enc.lengths.max()) == 32


@pytest.mark.parametrize("wid", [1, 2, 4])
def test_workload_single_matrix(codec, wid):
    x = workloads.matrix(wid, 0)
    m, enc = full_check(codec, x, call_oracle_decode=(wid == 1))
    assert m.stored_bytes == oracle.stored_bytes(enc)


@pytest.mark.parametrize("wid", [3, 5])
def test_workload_block_batched(codec, wid):
    """A whole transformer block: per-matrix codebooks, one decode launch
    (the bench configuration)."""
    names = [nm for nm, _ in workloads.WORKLOADS[wid][1]]
    mats, xs = [], []
    for i, _ in enumerate(names):
        x = workloads.matrix(wid, i).reshape(-1)
        enc = oracle.encode(x)
        m = codec.compress(to_dev(x))
        assert_encoded_equal(m, enc)
        mats.append(m)
        xs.append(x)
        del enc
    outs = codec.decompress_block(mats)
    for x, o in zip(xs, outs):
        assert np.array_equal(bits_of(o), x)


def test_decode_reports_corrupt_positions_without_fault(codec):
    x = workloads.random_bf16(2_000_000, seed=9)
    m = codec.compress(to_dev(x))
    pos = m.block_pos.clone()
    m.block_pos[3] += 5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codec.decompress(m, status=status)
    assert int(status.item()) == 4  # DF11_ERR_CORRUPT
    m.block_pos.copy_(pos)
    m.block_pos[5] = int(m.n) + 100  # beyond the matrix: must not be dereferenced
    status.zero_()
    codec.decompress(m, status=status)
    assert int(status.item()) == 4
    m.block_pos.copy_(pos)
    m.stream[1000:1010] ^= 0x5A  # flipped stream bits change the counts
    status.zero_()
    out = codec.decompress(m, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) in (0, 4)
    m.stream[1000:1010] ^= 0x5A
    status.zero_()
    out = codec.decompress(m, status=status)
    assert int(status.item()) == 0 and np.array_equal(bits_of(out), x)


def test_encode_reports_value_without_code(codec):
    import lossless_bf16_weight_df11_b200 as df11
    x = workloads.random_bf16(100_000, seed=4)
    st, cb = df11.df11_build_codebook(oracle.histogram(oracle.split(x[:50_000])[0]), 32)
    missing = [s for s in range(256) if cb.len[s] == 0]
    x[77] = (missing[0] << 7) | 1
    with pytest.raises(df11.DF11Error):
        codec.compress(to_dev(x), codebook=cb)
