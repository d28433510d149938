"""The .df11 container (df11_write / df11_read, include/df11.h): the oracle's
encoded arrays survive a write and a read byte for byte, the header fields and
section offsets follow the documented layout, the trailing checksum is the
standard CRC-32 (checked against zlib's), and every kind of damage is
reported as DF11_ERR_CORRUPT.  df11_codebook_from_lengths rebuilds the
oracle's canonical codes from the stored lengths.  The GPU tests decode
matrices that went through the container, bit for bit."""
import ctypes
import zlib

import numpy as np
import pytest

import lossless_bf16_weight_df11_b200 as df11
import oracle
import workloads

HDR = df11.FILE_HEADER_BYTES


@pytest.fixture(scope="module")
def lib():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    return df11.load()


def host_matrix(enc, shape=None, cap=11, max_block_codes=0):
    arrs = dict(lengths=np.ascontiguousarray(enc.lengths, np.uint8),
                gaps=np.ascontiguousarray(enc.gaps_packed, np.uint8),
                block_pos=np.ascontiguousarray(enc.block_pos, np.uint32),
                stream=np.ascontiguousarray(enc.stream, np.uint8),
                sign_mantissa=np.ascontiguousarray(enc.sign_mantissa, np.uint8))
    hm = df11.df11_host_matrix(n=enc.n, total_bits=enc.total_bits, cap=cap,
                               max_block_codes=max_block_codes)
    shape = shape or ()
    hm.ndim = len(shape)
    for i, d in enumerate(shape):
        hm.shape[i] = d
    for k, a in arrs.items():
        setattr(hm, k, a.ctypes.data)
    return hm, arrs


def write(enc, **kw):
    hm, arrs = host_matrix(enc, **kw)
    size = df11.df11_file_bytes(enc.n, enc.total_bits)
    buf = np.zeros(size, np.uint8)
    st, written = df11.df11_write(hm, buf.ctypes.data, size)
    assert st == 0 and written == size
    return buf


def read(buf):
    buf = np.ascontiguousarray(buf)
    st, hm = df11.df11_read(buf.ctypes.data, buf.size)
    return st, hm, buf


def r16(x):
    return (x + 15) // 16 * 16


def sections(n, total_bits):
    C = (total_bits + 63) // 64
    B = (C + 255) // 256
    gaps = HDR
    pos = r16(gaps + (5 * C + 7) // 8)
    stream = r16(pos + 4 * (B + 1))
    sm = r16(stream + 8 * C)
    crc = r16(sm + n)
    return gaps, pos, stream, sm, crc


CASES = {
    "workload1": lambda: workloads.matrix(1, 0).reshape(-1),
    "ragged_4097": lambda: workloads.random_bf16(4097, seed=7),
    "one_value": lambda: workloads.random_bf16(1, seed=8),
    "empty": lambda: workloads.random_bf16(0, seed=9),
    "patterns": workloads.all_patterns,
    "single_symbol": lambda: workloads.constant(70_001, 0x3F80),
}


@pytest.mark.parametrize("name", list(CASES))
def test_roundtrip_of_oracle_arrays(lib, name):
    x = CASES[name]()
    enc = oracle.encode(x, cap=11)
    shape = (x.size,) if x.size else ()
    buf = write(enc, shape=shape, max_block_codes=123)
    g, p, s, sm, crc = sections(enc.n, enc.total_bits)
    assert buf.size == crc + 4
    # header fields at their documented offsets
    assert bytes(buf[:4]) == b"DF11"
    v = buf[:HDR]
    assert int(v[4:8].view(np.uint32)[0]) == df11.FILE_VERSION
    assert int(v[8:16].view(np.uint64)[0]) == enc.n
    assert int(v[16:24].view(np.uint64)[0]) == enc.total_bits
    assert int(v[24:28].view(np.uint32)[0]) == 11 and int(v[28:32].view(np.uint32)[0]) == 123
    assert np.array_equal(buf[72:328], enc.lengths)
    assert not buf[328:HDR].any()
    # the sections, their zero padding, and the standard CRC-32 of the rest
    assert np.array_equal(buf[g:g + enc.gaps_packed.size], enc.gaps_packed)
    assert np.array_equal(buf[p:p + 4 * enc.block_pos.size].view(np.uint32), enc.block_pos)
    assert np.array_equal(buf[s:s + enc.stream.size], enc.stream)
    assert np.array_equal(buf[sm:sm + enc.n], enc.sign_mantissa)
    assert int(buf[crc:].view(np.uint32)[0]) == zlib.crc32(buf[:crc].tobytes())
    st, hm, b2 = read(buf)
    assert st == 0
    base = b2.ctypes.data
    assert (hm.gaps - base, hm.block_pos - base, hm.stream - base, hm.sign_mantissa - base) == \
        (g, p, s, sm)
    assert (hm.n, hm.total_bits, hm.cap, hm.max_block_codes) == (enc.n, enc.total_bits, 11, 123)
    assert hm.ndim == len(shape)


def test_file_size_formula(lib):
    for n, bits in [(0, 0), (1, 1), (10, 30), (4097, 4097 * 7), (1 << 20, 3 << 20)]:
        assert df11.df11_file_bytes(n, bits) == sections(n, bits)[4] + 4
    assert df11.df11_file_bytes(10, 5) == 0     # fewer bits than values
    assert df11.df11_file_bytes(10, 400) == 0   # more than 32 bits per value


def damaged(buf, where, xor=0x40):
    b = buf.copy()
    b[where] ^= xor
    return b


def test_damage_is_reported(lib):
    enc = oracle.encode(workloads.random_bf16(100_000, seed=3), cap=11)
    buf = write(enc, shape=(100_000,))
    g, p, s, sm, crc = sections(enc.n, enc.total_bits)
    corrupt = df11.DF11_ERR_CORRUPT
    assert read(buf)[0] == 0
    assert read(damaged(buf, 0))[0] == corrupt             # magic
    assert read(damaged(buf, 4))[0] == corrupt             # version
    assert read(damaged(buf, 9))[0] == corrupt             # n: sizes disagree
    assert read(buf[:-1])[0] == corrupt                    # truncated
    assert read(np.concatenate([buf, np.zeros(16, np.uint8)]))[0] == corrupt  # trailing bytes
    for where in (80, g + 3, p + 5, s + 100, sm + 7, crc):  # lengths, sections, checksum
        assert read(damaged(buf, where))[0] == corrupt, where
    # a well-formed container holding inconsistent metadata: df11_validate's checks
    bad = oracle.encode(workloads.random_bf16(100_000, seed=3), cap=11)
    bad.block_pos[3], bad.block_pos[4] = bad.block_pos[4], bad.block_pos[3]
    assert read(write(bad, shape=(100_000,)))[0] == corrupt


def test_write_rejects_bad_arguments(lib):
    enc = oracle.encode(workloads.random_bf16(1000, seed=4), cap=11)
    hm, arrs = host_matrix(enc, shape=(10, 99))         # 990 != 1000
    size = df11.df11_file_bytes(enc.n, enc.total_bits)
    buf = np.zeros(size, np.uint8)
    assert df11.df11_write(hm, buf.ctypes.data, size)[0] == df11.DF11_ERR_INVALID_ARG
    hm, arrs = host_matrix(enc, shape=(10, 100))
    assert df11.df11_write(hm, buf.ctypes.data, size - 1)[0] == df11.DF11_ERR_INVALID_ARG
    over = arrs["lengths"].copy()
    over[over > 0] = 1                                    # Kraft sum > 1
    hm.lengths = over.ctypes.data
    assert df11.df11_write(hm, buf.ctypes.data, size)[0] == df11.DF11_ERR_INVALID_ARG


def hist_from(counts, first):
    h = np.zeros(256, np.uint64)
    h[first:first + len(counts)] = counts
    return h


@pytest.mark.parametrize("h", [
    hist_from([1000, 300, 100, 30, 10, 3, 1], 120),
    hist_from(workloads.fibonacci_counts(34), 100),
    np.ones(256, np.uint64),
    hist_from([5], 77),
    hist_from([1, 1], 0),
], ids=["skew", "fibonacci34", "uniform", "one", "two"])
def test_codebook_from_lengths_is_canonical(lib, h):
    ln, code = oracle.codebook(h)
    lens = np.ascontiguousarray(ln, np.uint8)
    st, cb = df11.df11_codebook_from_lengths(lens.ctypes.data, 32)
    assert st == 0
    assert list(cb.len) == ln.tolist() and list(cb.code) == code.tolist()
    nz = ln[ln > 0]
    assert (cb.max_len, cb.min_len, cb.n_symbols) == (nz.max(), nz.min(), nz.size)


def test_codebook_from_lengths_rejects(lib):
    lens = np.zeros(256, np.uint8)
    lens[:3] = 1                                          # three 1-bit codes
    assert df11.df11_codebook_from_lengths(lens.ctypes.data, 32)[0] == df11.DF11_ERR_INVALID_ARG
    lens[:] = 0
    lens[0] = 33
    assert df11.df11_codebook_from_lengths(lens.ctypes.data, 32)[0] == df11.DF11_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["workload1", "ragged_4097", "patterns", "single_symbol"])
def test_gpu_decode_after_the_container(lib, name, tmp_path):
    import torch
    import lossless_bf16_weight_df11_b200.codec as codec
    x = CASES[name]()
    w = torch.from_numpy(x.view(np.int16)).cuda()
    for cap in (11, 32):
        m = codec.compress(w, cap=cap)
        path = str(tmp_path / f"{name}_{cap}.df11")
        nbytes = codec.save(path, m)
        assert nbytes == df11.df11_file_bytes(m.n, m.total_bits)
        m2 = codec.load(path, "cuda")
        assert m2.max_block_codes == m.max_block_codes and m2.shape == m.shape
        got = codec.decompress(m2).reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, x)
        # a container written from the oracle's arrays decodes the same way
        enc = oracle.encode(x, cap=cap)
        m3 = codec.deserialize(write(enc, shape=(x.size,), cap=cap), "cuda")
        got3 = codec.decompress(m3).reshape(-1).view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got3, x)
