"""CPU tests of the host side of the pipelined host-buffer decode
(df11_decode_host_scratch_bytes, and the checks df11_decode_host_batch makes
before it queues anything): how matrices are cut into pieces, and which
metadata is rejected on the host.  Only host memory is read; every batch
call here fails its host checks, so no device pointer is ever used."""
import numpy as np
import pytest

import lossless_bf16_weight_df11_b200 as df11
from lossless_bf16_weight_df11_b200 import build as df11_build

BLOCK_BITS = 64 * 256
FIRST = 256           # the call's first piece, in blocks
PIECE_BLOCKS = 4096   # the longest piece (each piece may double the one before)
RAMP = sum(FIRST << k for k in range(5))  # 256 + 512 + ... + 4096
ALIGN = 256


@pytest.fixture(scope="module")
def lib():
    df11_build.build()
    return df11.load()


class Fake:
    """A host matrix whose metadata the host side reads (lengths and block
    positions); the byte arrays are zero-filled buffers of the right sizes."""

    def __init__(self, blocks: int, per_block: int, lengths=(2, 2, 2, 3, 3), tail_bits=100):
        self.total_bits = blocks * BLOCK_BITS - tail_bits
        self.pos = np.arange(blocks + 1, dtype=np.uint32) * per_block
        self.n = int(self.pos[-1])
        self.lengths = np.zeros(256, np.uint8)
        self.lengths[: len(lengths)] = lengths
        st, z = df11.df11_sizes_from_bits(self.n, self.total_bits)
        assert st == 0
        self.sizes = z
        self.stream = np.zeros(z.stream_bytes, np.uint8)
        self.gaps = np.zeros(z.gaps_bytes, np.uint8)
        self.sm = np.zeros(max(1, self.n), np.uint8)

    def abi(self):
        return df11.df11_host_matrix(
            n=self.n, total_bits=self.total_bits, cap=32, max_block_codes=0, ndim=0,
            lengths=self.lengths.ctypes.data, gaps=self.gaps.ctypes.data,
            block_pos=self.pos.ctypes.data, stream=self.stream.ctypes.data,
            sign_mantissa=self.sm.ctypes.data)


def scratch(fakes):
    return df11.df11_decode_host_scratch_bytes([f.abi() for f in fakes])


def test_one_piece_sized_by_the_largest(lib):
    small, large = Fake(10, 3000), Fake(40, 3000)
    s_small, s_large = scratch([small]), scratch([large])
    assert s_small > 0 and s_large > s_small
    # one matrix's tables more, the slots sized by the larger matrix
    both = scratch([small, large])
    assert 0 < both - s_large <= df11.df11_tables_bytes() + 2 * ALIGN
    assert scratch([large, small]) == both


def test_slots_grow_with_the_piece_then_stop(lib):
    # pieces of 256, 512, ..., 4096 blocks: the slot no longer grows after
    one = scratch([Fake(RAMP, 3000)])
    assert one == scratch([Fake(RAMP + 2 * PIECE_BLOCKS + 100, 3000)])
    assert one > scratch([Fake(RAMP - 2, 3000)])  # its last piece is 4094 blocks
    # a matrix of one first piece
    assert scratch([Fake(FIRST - 2, 3000)]) < scratch([Fake(FIRST, 3000)])


def test_pieces_double_across_matrices(lib):
    # the ramp runs over the call, not per matrix: after a first matrix of
    # one full first piece, a second matrix starts with a piece of 512 blocks
    a, b = Fake(FIRST, 3000), Fake(2 * FIRST + 2, 3000)
    assert scratch([a, b]) > scratch([b, a])


def test_no_tail_of_one_block(lib):
    # FIRST + 1 blocks: the last block joins the first piece
    assert scratch([Fake(FIRST + 1, 3000)]) > scratch([Fake(FIRST, 3000)])
    # FIRST + 2 blocks: two pieces, the first of FIRST blocks
    assert scratch([Fake(FIRST + 2, 3000)]) == scratch([Fake(FIRST, 3000)])


def test_cut_moves_on_where_a_piece_would_be_too_short(lib):
    """A piece must hold at least min_len bits per value.  With every code 2
    bits long a block holds 8192 of them; one more position at the cut (a
    code running over it) would break that, so the cut moves on a unit."""
    two = dict(lengths=(2, 2, 2, 2), tail_bits=0)
    f = Fake(FIRST + 10, 8192, **two)
    base = scratch([f])
    assert base == scratch([Fake(FIRST, 8192, **two)])
    f.pos[FIRST] += 1
    moved = scratch([f])
    # the first piece now ends at FIRST + 2: longer than one of FIRST + 1
    # blocks (a matrix that stays one piece)
    assert moved > scratch([Fake(FIRST + 1, 8192, **two)]) > base


def test_metadata_rejected_on_the_host(lib):
    f = Fake(20, 1000)
    out = np.zeros(f.n, np.uint16)
    need = scratch([f])
    fake_dev = 1 << 40  # never used: every call below fails its host checks

    def call(m, size=need, outs=None):
        return df11.df11_decode_host_batch([m.abi()], [out.ctypes.data] if outs is None else outs,
                                           fake_dev, size, fake_dev, 0)

    assert call(f, need - 1) == df11.DF11_ERR_INVALID_ARG
    assert call(f, outs=[0]) == df11.DF11_ERR_INVALID_ARG
    f.pos[0] = 1
    assert call(f) == df11.DF11_ERR_CORRUPT and scratch([f]) == 0
    f.pos[0] = 0
    f.pos[-1] += 1
    assert call(f) == df11.DF11_ERR_CORRUPT and scratch([f]) == 0
    f.pos[-1] -= 1
    f.lengths[:] = 0
    f.lengths[:3] = 1  # over-full code
    assert call(f) == df11.DF11_ERR_INVALID_ARG
    f.lengths[:] = 0
    f.lengths[:256] = 8
    f.lengths[0] = 0
    f.lengths[1:3] = 9  # shortest code 8 bits: accepted
    assert scratch([f]) > 0
    f.lengths[:] = 9  # shortest code 9 bits: no complete code has one
    assert call(f) == df11.DF11_ERR_INVALID_ARG and scratch([f]) == 0
    bad = Fake(4, 3000)
    bad.total_bits = bad.n * 33
    assert scratch([bad]) == 0
    assert df11.df11_decode_host_batch([], [], fake_dev, 0, fake_dev, 0) == 0
