"""GPU parity of the rANS exponent-codec variant against the oracle.

Encode: the device's stream, unit offsets and sign/mantissa plane equal the
oracle's byte for byte.  Decode: the device decodes the oracle's encoding
(uploaded as is) and its own back to the input bit for bit.  Corrupt
metadata is reported and nothing outside the output is written.  Sizes span
ragged units, several units per CTA, matrices whose segments overflow the
decoder's shared-memory word buffers (uniform exponents: ~1024 words per
segment), batches of more matrices than one launch takes, and the full
8192 x 28672 matrix of the Llama-3-70B-shaped block."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rans():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    import lossless_bf16_weight_df11_b200.rans as r
    return r


@pytest.fixture(scope="module")
def df11(rans):
    import lossless_bf16_weight_df11_b200 as m
    return m


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda()


def assert_encoding_equal(m, enc):
    h = m.host_arrays()
    assert np.array_equal(h["freq"], enc.freq)
    assert np.array_equal(h["off16"], enc.off16)
    assert np.array_equal(h["stream"], enc.stream)
    assert np.array_equal(h["sign_mantissa"], enc.sign_mantissa)


def cases():
    return [
        ("one", lambda: workloads.random_bf16(1, seed=1)),
        ("31", lambda: workloads.random_bf16(31, seed=2)),
        ("33", lambda: workloads.random_bf16(33, seed=3)),
        ("2049", lambda: workloads.random_bf16(2049, seed=4)),
        ("16383", lambda: workloads.random_bf16(16383, seed=5)),
        ("16384", lambda: workloads.random_bf16(16384, seed=6)),
        ("16385", lambda: workloads.random_bf16(16385, seed=7)),
        ("1000003", lambda: workloads.random_bf16(1_000_003, seed=8)),
        ("all_patterns_shuffled", lambda: workloads.shuffled_patterns(copies=3, seed=9)),
        ("fibonacci_rare", lambda: workloads.fibonacci_exponents(30)[: 3 * 16384 + 999]),
        ("single_symbol", lambda: workloads.constant(70_000, 0x3F80)),
        ("matrix_4096x4096", lambda: workloads.matrix(2, 0)),
    ]


@pytest.mark.parametrize("name,gen", cases(), ids=[c[0] for c in cases()])
def test_encode_matches_oracle_and_decodes(rans, name, gen):
    x = np.ascontiguousarray(gen(), np.uint16).reshape(-1)
    enc = oracle.rans_encode(x)
    m = rans.compress(to_dev(x))
    torch.cuda.synchronize()
    assert_encoding_equal(m, enc)
    y = rans.decompress(m)
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), x)
    # the oracle's own arrays, uploaded, decode on the device as well
    mo = rans.from_host_arrays(x.shape, x.size, enc.freq, enc.stream, enc.off16, enc.sign_mantissa,
                               "cuda")
    yo = rans.decompress(mo)
    assert np.array_equal(yo.view(torch.int16).cpu().numpy().view(np.uint16), x)


def test_given_frequencies_hand_example(rans):
    """The hand-derived renormalisation example (frequencies 4094/1/1)."""
    e = np.full(65, 127, np.uint32)
    e[0], e[32], e[64] = 128, 128, 129
    i = np.arange(65, dtype=np.uint32)
    x = (((i & 1) << 15) | (e << 7) | (i * 37 % 128)).astype(np.uint16)
    f = np.zeros(256, np.uint32)
    f[127], f[128], f[129] = 4094, 1, 1
    enc = oracle.rans_encode(x, freq=f)
    m = rans.compress(to_dev(x), freq=f)
    assert_encoding_equal(m, enc)
    assert m.stream_bytes == 160
    y = rans.decompress(m)
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), x)


def test_uniform_frequencies_take_the_unstaged_path(rans):
    """f = 16 for every exponent: ~1024 words per 64-step segment, more than a
    staging buffer holds, so every segment reads its words from global memory."""
    x = workloads.shuffled_patterns(copies=2, seed=3)
    enc = oracle.rans_encode(x)
    spans = []
    for u in range(enc.units):
        p = enc.stream[16 * enc.off16[u]: 16 * enc.off16[u] + 144].view(np.uint16)[64:72]
        words = (16 * int(enc.off16[u + 1] - enc.off16[u]) - 144) // 2
        spans.append(np.diff(np.append(p.astype(np.int64), words)).min())
    assert min(spans) > 512
    m = rans.compress(to_dev(x))
    assert_encoding_equal(m, enc)
    y = rans.decompress(m)
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), x)


def test_exponent_without_frequency_is_reported(rans, df11):
    x = workloads.random_bf16(40_000, seed=12)
    f = oracle.rans_freqs(oracle.histogram(oracle.split(x)[0]))
    s = int(np.flatnonzero(f)[-1])
    f2 = f.copy()
    f2[int(np.flatnonzero(f)[0])] += f2[s]
    f2[s] = 0
    with pytest.raises(df11.DF11Error) as ei:
        rans.compress(to_dev(x), freq=f2)
    assert ei.value.status == df11.DF11_ERR_SYMBOL_NOT_IN_CODEBOOK


def corrupt_copy(rans, m, where):
    h = m.host_arrays()
    s, off = h["stream"].copy(), h["off16"].copy()
    p = 16 * int(off[1])                      # unit 1
    if where == "state":
        s[p + 4 * 7] ^= 0x10
    elif where == "word":
        s[p + 144 + 2 * 40] ^= 0x04
    elif where == "segment_start":
        s[p + 128 + 2 * 5] ^= 0x01
    elif where == "off16_order":
        off[2] = off[1] - 1
    elif where == "off16_past_end":
        off[-2] = off[-1] + 5
    return rans.from_host_arrays(m.shape, m.n, h["freq"], s, off, h["sign_mantissa"], "cuda")


@pytest.mark.parametrize("where", ["state", "word", "segment_start", "off16_order",
                                   "off16_past_end"])
def test_corruption_reported_and_writes_stay_in_the_output(rans, df11, where):
    x = workloads.random_bf16(5 * 16384 + 100, seed=13)
    m = rans.compress(to_dev(x))
    bad = corrupt_copy(rans, m, where)
    guard = 4096
    full = torch.full((x.size + 2 * guard,), 0x5A5A, dtype=torch.int16, device="cuda")
    out = full[guard: guard + x.size]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rans.decompress_block([bad], [out.view(torch.bfloat16)], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == df11.DF11_ERR_CORRUPT
    f = full.cpu().numpy()
    assert (f[:guard] == 0x5A5A).all() and (f[guard + x.size:] == 0x5A5A).all()


def test_batch_larger_than_one_launch_with_empty_matrices(rans):
    shapes = [(0,)] + [(1000 + 5000 * i,) for i in range(40)] + [(0,)]
    xs = [workloads.random_bf16(s[0], seed=300 + i) for i, s in enumerate(shapes)]
    ms = rans.compress_block([to_dev(x) for x in xs])
    outs = rans.decompress_block(ms)
    for x, y in zip(xs, outs):
        assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), x)


def test_llama3_70b_block_down_projection_full_size(rans):
    """The largest matrix of the bench's block (8192 x 28672, 235 M values):
    every byte of the encoding against the oracle, and the decode against
    the input (the oracle's round trip is the identity)."""
    x = workloads.matrix(5, 6).reshape(-1)
    m = rans.compress(to_dev(x))
    enc = oracle.rans_encode(x)
    assert_encoding_equal(m, enc)
    del enc
    y = rans.decompress(m)
    assert torch.equal(y.view(torch.int16).reshape(-1), to_dev(x))


def test_decode_is_repeatable_in_a_batch_of_the_block(rans):
    names = workloads.WORKLOADS[3][1]
    xs = [workloads.matrix(3, i).reshape(-1) for i in range(len(names))]
    ms = rans.compress_block([to_dev(x) for x in xs])
    for _ in range(2):
        outs = rans.decompress_block(ms)
        for x, y in zip(xs, outs):
            assert torch.equal(y.view(torch.int16).reshape(-1), to_dev(x))


GUARD = 4096   # bytes on each side, a multiple of 16
PATTERN = 0xA5


class Guarded:
    def __init__(self, nbytes, fill=PATTERN):
        self.nbytes = int(nbytes)
        self.full = torch.full((self.nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.inner = self.full[GUARD:GUARD + self.nbytes]
        if fill != PATTERN:
            self.inner.fill_(fill)

    @property
    def ptr(self):
        return self.inner.data_ptr()

    def margins_intact(self):
        f = self.full.cpu().numpy()
        return bool((f[:GUARD] == PATTERN).all() and (f[GUARD + self.nbytes:] == PATTERN).all())


@pytest.mark.parametrize("name,gen", [
    ("fibonacci_rare", lambda: workloads.fibonacci_exponents(30)[: 3 * 16384 + 999]),
    ("ragged_16385", lambda: workloads.random_bf16(16385, seed=21)),
    ("uniform_unstaged", lambda: workloads.shuffled_patterns(copies=1, seed=5)),
    ("seventeen", lambda: workloads.random_bf16(17, seed=22)),
], ids=lambda v: v if isinstance(v, str) else "")
def test_encode_and_decode_stay_inside_their_buffers(df11, name, gen):
    """Every buffer of the C ABI calls sits between guard bands: encode
    writes only its outputs (exactly the format's bytes), decode only its
    output, and neither touches its inputs."""
    x = np.ascontiguousarray(gen(), np.uint16).reshape(-1)
    n = x.size
    units = df11.df11_rans_units(n)
    w = Guarded(2 * n)
    w.inner.copy_(torch.from_numpy(x.view(np.uint8).copy()).cuda())
    hist = torch.empty(256, dtype=torch.int64, device="cuda")
    df11.check(df11.df11_histogram(w.ptr, n, hist.data_ptr(), 0))
    st, freq = df11.df11_rans_freqs(hist.cpu().numpy().view(np.uint64))
    df11.check(st)
    host_t = np.zeros(df11.RANS_TABLES_BYTES, np.uint8)
    df11.check(df11.df11_rans_build_tables(freq, host_t.ctypes.data, host_t.size))
    tables = Guarded(host_t.size)
    tables.inner.copy_(torch.from_numpy(host_t).cuda())
    uw, off = Guarded(4 * units, fill=0x5A), Guarded(4 * (units + 1), fill=0x5A)
    status = Guarded(16, fill=0)
    df11.check(df11.df11_rans_encode_sizes(w.ptr, n, tables.ptr, uw.ptr, off.ptr, status.ptr, 0))
    torch.cuda.synchronize()
    total16 = int(off.inner.cpu().numpy().view(np.uint32)[units])
    stream, sm = Guarded(16 * total16, fill=0x5A), Guarded(n, fill=0x5A)
    df11.check(df11.df11_rans_encode(w.ptr, n, tables.ptr, uw.ptr, off.ptr, stream.ptr, sm.ptr,
                                     status.ptr, 0))
    torch.cuda.synchronize()
    assert int(status.inner.cpu().numpy().view(np.uint32)[0]) == 0
    for g, what in ((w, "input"), (tables, "tables"), (uw, "unit words"), (off, "off16"),
                    (stream, "stream"), (sm, "sign/mantissa"), (status, "status")):
        assert g.margins_intact(), f"encode wrote outside {what}"
    enc = oracle.rans_encode(x)
    assert np.array_equal(stream.inner.cpu().numpy(), enc.stream)
    assert np.array_equal(off.inner.cpu().numpy().view(np.uint32), enc.off16)
    assert np.array_equal(sm.inner.cpu().numpy(), enc.sign_mantissa)
    before = {k: g.full.clone() for k, g in (("stream", stream), ("off16", off), ("sm", sm),
                                               ("tables", tables))}
    out = Guarded(2 * n, fill=0)
    st2 = Guarded(16, fill=0)
    m = df11.df11_rans_matrix(n=n, stream=stream.ptr, off16=off.ptr, sign_mantissa=sm.ptr,
                              tables=tables.ptr)
    df11.check(df11.df11_rans_decode_batch([m], [out.ptr], st2.ptr, 0))
    torch.cuda.synchronize()
    assert int(st2.inner.cpu().numpy().view(np.uint32)[0]) == 0
    assert out.margins_intact() and st2.margins_intact()
    for k, g in (("stream", stream), ("off16", off), ("sm", sm), ("tables", tables)):
        assert torch.equal(g.full, before[k]), f"decode modified its input {k}"
    assert np.array_equal(out.inner.cpu().numpy().view(np.uint16), x)
