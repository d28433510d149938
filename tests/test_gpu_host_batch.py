"""The decode from host memory to host memory (df11_decode_host_batch): the
oracle's encodings, held in page-locked host buffers, decoded through the
pipelined call and compared bit for bit with the words the oracle encoded
(the oracle's round trip is the identity, pinned in test_oracle_pins.py).
Matrices of different sizes, and the pieces a large matrix is cut into, take
turns in the scratch slots; an empty matrix, a single-symbol one, all 65,536
bit patterns, ragged tails and a matrix of two pieces are among them.  The
full-size case encodes on the GPU (parity-tested against the oracle
elsewhere) and checks the round trip of the Llama-3-8B-shaped block."""
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


def pinned(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a).reshape(-1).view(np.uint8)
    t = torch.empty(a.size, dtype=torch.uint8, pin_memory=True)
    t.copy_(torch.from_numpy(a))
    return t


def host_from(codec, enc, cap=11):
    arrays = {"stream": pinned(enc.stream), "gaps": pinned(enc.gaps_packed),
              "block_pos": pinned(enc.block_pos.astype(np.uint32)),
              "sign_mantissa": pinned(enc.sign_mantissa), "lengths": pinned(enc.lengths)}
    return codec.HostMatrix((enc.n,), enc.n, enc.total_bits, cap, 0, arrays)


def host_matrix(codec, x: np.ndarray, cap: int):
    """The oracle's encoding of x as a HostMatrix (no GPU step involved)."""
    enc = oracle.encode(np.ascontiguousarray(x, np.uint16).reshape(-1), cap=cap)
    return host_from(codec, enc, cap)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.reshape(-1).view(torch.int16).numpy().view(np.uint16)


def mixed_block():
    return [workloads.random_bf16(262_144, seed=1),
            workloads.random_bf16(4097, seed=2),
            workloads.all_patterns(),
            np.zeros(0, np.uint16),
            workloads.constant(70_001),
            workloads.random_bf16(1_500_000, seed=3, std=0.5),
            workloads.fibonacci_exponents(26)[:100_000],
            workloads.random_bf16(1, seed=4)]


@pytest.mark.parametrize("cap", [11, 12, 32])
def test_mixed_block_matches_the_oracle(codec, cap):
    xs = mixed_block()
    hms = [host_matrix(codec, x, cap) for x in xs]
    outs = codec.decompress_host(hms)
    for i, (o, x) in enumerate(zip(outs, xs)):
        assert np.array_equal(bits(o), x), f"matrix {i}"


@pytest.fixture(scope="module")
def several_pieces():
    """13 M values, about 2,060 blocks: a matrix of several pieces (the
    call's first piece is 256 blocks long, each later one at most twice the
    one before)."""
    x = workloads.random_bf16(13_000_000, seed=50)
    return x, oracle.encode(x, cap=11)


def test_matrix_of_several_pieces(codec, several_pieces):
    x, enc = several_pieces
    assert enc.n_blocks > 256 + 512 + 1024 + 2
    small = workloads.random_bf16(50_000, seed=51)
    hms = [host_matrix(codec, small, 11), host_from(codec, enc), host_matrix(codec, small, 11)]
    outs = codec.decompress_host(hms)
    assert np.array_equal(bits(outs[1]), x)
    assert np.array_equal(bits(outs[0]), small) and np.array_equal(bits(outs[2]), small)


def test_corrupt_position_at_a_cut(codec, several_pieces):
    """Positions moved at the cut between two pieces: both pieces disagree
    with their streams, the device reports it, nothing is written outside the
    output."""
    x, enc = several_pieces
    h = host_from(codec, enc)
    pos = h.arrays["block_pos"].view(torch.int32)
    keep = pos.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for v in (5, -5):
        pos.copy_(keep)
        pos[256] += v  # the first cut
        status.zero_()
        codec.decompress_host([h], status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 4  # DF11_ERR_CORRUPT
    pos.copy_(keep)
    status.zero_()
    outs = codec.decompress_host([h], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and np.array_equal(bits(outs[0]), x)


def test_caller_stream_and_reused_scratch(codec):
    """Work queued on a side stream: a synchronize of that stream alone makes
    the host outputs ready; the same scratch serves a second call."""
    xs = [workloads.random_bf16(n, seed=20 + n % 7) for n in (300_000, 5, 1_000_003, 65_536)]
    hms = [host_matrix(codec, x, 11) for x in xs]
    scratch = codec.host_scratch(hms, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    for rep in range(2):
        outs = [torch.full(x.shape, float("nan"), dtype=torch.bfloat16).pin_memory() for x in xs]
        codec.decompress_host(hms, outs, scratch=scratch, status=status, stream=s)
        s.synchronize()
        assert int(status.item()) == 0
        for o, x in zip(outs, xs):
            assert np.array_equal(bits(o), x), rep


def test_pageable_host_buffers(codec):
    xs = [workloads.random_bf16(200_000, seed=30), workloads.random_bf16(33, seed=31)]
    hms = [host_matrix(codec, x, 11) for x in xs]
    for h in hms:
        h.arrays = {k: v.clone() for k, v in h.arrays.items()}  # ordinary host memory
        assert not h.arrays["stream"].is_pinned()
    outs = [torch.empty(x.shape, dtype=torch.bfloat16) for x in xs]
    codec.decompress_host(hms, outs)
    for o, x in zip(outs, xs):
        assert np.array_equal(bits(o), x)


def test_arguments_are_checked_before_anything_is_queued(codec):
    from lossless_bf16_weight_df11_b200 import (DF11_ERR_INVALID_ARG, df11_decode_host_batch,
                                                df11_decode_host_scratch_bytes)
    xs = [workloads.random_bf16(10_000, seed=40), workloads.random_bf16(50_000, seed=41)]
    hms = [host_matrix(codec, x, 11) for x in xs]
    abis = [h.abi() for h in hms]
    need = df11_decode_host_scratch_bytes(abis)
    assert need > 2 * 2 * 50_000
    scratch = torch.zeros(need + 512, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = [torch.empty(x.shape, dtype=torch.bfloat16, pin_memory=True) for x in xs]
    ptrs = [o.data_ptr() for o in outs]
    base = scratch.data_ptr()
    assert df11_decode_host_batch(abis, ptrs, base, need - 1, status.data_ptr()) == \
        DF11_ERR_INVALID_ARG
    assert df11_decode_host_batch(abis, ptrs, base + 16, need, status.data_ptr()) == \
        DF11_ERR_INVALID_ARG
    assert df11_decode_host_batch(abis, ptrs, base, need, 0) == DF11_ERR_INVALID_ARG
    assert df11_decode_host_batch(abis, [ptrs[0], 0], base, need, status.data_ptr()) == \
        DF11_ERR_INVALID_ARG
    bad = hms[1].abi()
    bad.total_bits = 50_000 * 32 + 1  # more code bits than 32 per value
    assert df11_decode_host_scratch_bytes([abis[0], bad]) == 0
    lens = hms[0].arrays["lengths"].clone()
    hms[0].arrays["lengths"][:3] = 1  # over-full code (Kraft sum > 1)
    assert df11_decode_host_batch([hms[0].abi()], ptrs[:1], base, need, status.data_ptr()) == \
        DF11_ERR_INVALID_ARG
    hms[0].arrays["lengths"].copy_(lens)
    assert df11_decode_host_batch([], [], base, need, status.data_ptr()) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert df11_decode_host_batch(abis, ptrs, base, need, status.data_ptr()) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for o, x in zip(outs, xs):
        assert np.array_equal(bits(o), x)


def test_corrupt_positions_are_reported_without_fault(codec):
    x = workloads.random_bf16(2_000_000, seed=9)
    good = host_matrix(codec, x, 11)
    other = host_matrix(codec, workloads.random_bf16(100_000, seed=8), 11)
    pos = good.arrays["block_pos"].view(torch.int32)
    keep = pos.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for b, v in ((3, int(keep[3]) + 5), (5, good.n + 100)):
        pos.copy_(keep)
        pos[b] = v
        status.zero_()
        codec.decompress_host([other, good], status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 4  # DF11_ERR_CORRUPT
    pos.copy_(keep)
    status.zero_()
    outs = codec.decompress_host([other, good], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and np.array_equal(bits(outs[1]), x)


def test_llama3_8b_block_full_size(codec):
    """Workload 3 at full size (7 matrices, 218 M weights), encoded on the
    GPU, round trip through host memory."""
    ws = [torch.from_numpy(workloads.matrix(3, i).reshape(-1).view(np.int16)).cuda()
          for i in range(len(workloads.workload_sizes(3)))]
    ms = codec.compress_block(ws)
    hms = [codec.HostMatrix.from_matrix(m) for m in ms]
    del ms
    outs = codec.decompress_host(hms)
    for o, w in zip(outs, ws):
        assert torch.equal(o.view(torch.int16).reshape(-1).cuda(), w)
