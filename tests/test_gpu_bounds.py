"""Encode and decode write nothing outside the buffers the format defines.

Every device buffer handed to the C ABI sits inside a larger allocation whose
margins (guard bands) hold a fixed byte pattern.  After df11_encode (and
df11_encode_static_ws) the margins of every output and of the workspace and
status words must still hold the pattern; df11_decode_block_batch must leave
its inputs (stream, gaps, block positions, sign/mantissa plane, tables) and
the margins of its outputs untouched (with no index, the run index or the
segment index; each index is built into a guarded buffer of its own).  The
decoded words are compared with the input, and the encoded arrays with the
oracle.

Inputs: the cases whose sizes exercise the most paths -- codes longer than
the decode table (cap 32), an odd number of blocks (a last work unit of one
block), a single symbol (1-bit codes), a handful of values, and the 4096 x
4096 workload matrix, whose block count gives every decode CTA several units.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

GUARD = 4096   # bytes on each side; a multiple of 16 keeps every pointer aligned
PATTERN = 0xA5


@pytest.fixture(scope="module")
def df11():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    import lossless_bf16_weight_df11_b200 as m
    return m


class Guarded:
    """nbytes usable bytes between two GUARD-byte margins of PATTERN."""

    def __init__(self, nbytes: int, dev, fill: int = PATTERN):
        self.nbytes = int(nbytes)
        self.full = torch.full((self.nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device=dev)
        self.inner = self.full[GUARD:GUARD + self.nbytes]
        if fill != PATTERN:
            self.inner.fill_(fill)

    @property
    def ptr(self) -> int:
        return self.inner.data_ptr()

    def margins_intact(self) -> bool:
        f = self.full.cpu().numpy()
        return bool((f[:GUARD] == PATTERN).all() and (f[GUARD + self.nbytes:] == PATTERN).all())


def _cases():
    return [
        ("fibonacci_cap32", lambda: workloads.fibonacci_exponents(34), 32),
        ("matrix_4096x4096_cap11", lambda: workloads.matrix(2, 0), 11),
        ("matrix_4096x4096_cap12", lambda: workloads.matrix(2, 0), 12),
        ("random_1000003_cap11", lambda: workloads.random_bf16(1_000_003, seed=2003), 11),
        ("random_1000003_cap32", lambda: workloads.random_bf16(1_000_003, seed=2004), 32),
        ("single_symbol_65537", lambda: workloads.constant(65_537, 0x3F80), 11),
        ("seventeen_values", lambda: workloads.random_bf16(17, seed=5), 11),
    ]


def _encode_guarded(df11, x: np.ndarray, cap: int, static_ws: bool):
    dev = torch.device("cuda", 0)
    n = x.size
    w = Guarded(max(2 * n, 16), dev)
    w.inner[: 2 * n].copy_(torch.from_numpy(x.view(np.uint8)).to(dev))
    stream = torch.cuda.current_stream().cuda_stream
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    df11.check(df11.df11_histogram(w.ptr, n, hist.data_ptr(), stream), "df11_histogram")
    h = hist.cpu().numpy().view(np.uint64)
    st, cb = df11.df11_build_codebook(h, cap)
    df11.check(st, "df11_build_codebook")
    st, sizes = df11.df11_encoded_sizes(cb, h, n)
    df11.check(st, "df11_encoded_sizes")
    bufs = {name: Guarded(getattr(sizes, name + "_alloc"), dev, fill=0x5A)
            for name in ("stream", "gaps", "block_pos", "sign_mantissa")}
    status = Guarded(16, dev, fill=0)  # [status, most codes per block, unused...]
    abi = df11.df11_encoded(stream=bufs["stream"].ptr, gaps=bufs["gaps"].ptr,
                            block_pos=bufs["block_pos"].ptr,
                            sign_mantissa=bufs["sign_mantissa"].ptr,
                            block_max=status.ptr + 4)
    ws = None
    if static_ws:
        df11.check(df11.df11_encode_static_ws(w.ptr, n, cb, sizes.total_bits, abi, status.ptr,
                                              stream), "df11_encode_static_ws")
    else:
        ws = Guarded(max(16, sizes.workspace_bytes), dev)
        df11.check(df11.df11_encode(w.ptr, n, cb, sizes.total_bits, abi, ws.ptr, ws.nbytes,
                                    status.ptr, stream), "df11_encode")
    torch.cuda.synchronize()
    st_words = status.inner.cpu().numpy().view(np.uint32)
    assert st_words[0] == 0, "device status"
    for name, g in bufs.items():
        assert g.margins_intact(), f"encode wrote outside {name}"
    assert status.margins_intact(), "encode wrote outside the status words"
    if ws is not None:
        assert ws.margins_intact(), "encode wrote outside the workspace"
    assert w.margins_intact(), "encode wrote into its input's margins"
    return cb, sizes, bufs, int(st_words[1])


@pytest.mark.parametrize("static_ws", [False, True])
@pytest.mark.parametrize("name,gen,cap", _cases())
def test_encode_and_decode_stay_inside_their_buffers(df11, name, gen, cap, static_ws):
    x = np.ascontiguousarray(gen(), np.uint16).reshape(-1)
    dev = torch.device("cuda", 0)
    cb, sizes, bufs, block_max = _encode_guarded(df11, x, cap, static_ws)
    enc = oracle.encode(x, cap=cap)
    assert np.array_equal(bufs["stream"].inner[: sizes.stream_bytes].cpu().numpy(), enc.stream)
    assert np.array_equal(bufs["gaps"].inner[: sizes.gaps_bytes].cpu().numpy(), enc.gaps_packed)
    assert np.array_equal(bufs["block_pos"].inner[: 4 * (sizes.n_blocks + 1)].cpu().numpy()
                          .view(np.uint32), enc.block_pos)
    if static_ws:
        return  # the decode half does not depend on which encoder ran
    tables = Guarded(sizes.tables_bytes, dev)
    host = np.zeros(sizes.tables_bytes, np.uint8)
    df11.check(df11.df11_build_tables(cb, host.ctypes.data, host.size), "df11_build_tables")
    tables.inner.copy_(torch.from_numpy(host).to(dev))
    before = {k: g.full.clone() for k, g in bufs.items()}
    before["tables"] = tables.full.clone()
    n = x.size
    sh = torch.cuda.current_stream().cuda_stream
    m = df11.df11_matrix(n=n, total_bits=sizes.total_bits, stream=bufs["stream"].ptr,
                         gaps=bufs["gaps"].ptr, block_pos=bufs["block_pos"].ptr,
                         sign_mantissa=bufs["sign_mantissa"].ptr, tables=tables.ptr,
                         min_len=max(1, cb.min_len), max_block_codes=block_max)
    # the run index, built into its own guarded buffer
    ri = Guarded(max(16, sizes.run_index_bytes), dev)
    ri_status = Guarded(16, dev, fill=0)
    df11.check(df11.df11_build_run_index(m, ri.ptr, ri_status.ptr, sh), "df11_build_run_index")
    torch.cuda.synchronize()
    assert int(ri_status.inner.cpu().numpy().view(np.uint32)[0]) == 0, "run index status"
    assert ri.margins_intact() and ri_status.margins_intact(), "run index wrote outside its buffers"
    for k, g in list(bufs.items()) + [("tables", tables)]:
        assert torch.equal(g.full, before[k]), f"the run index modified its input {k}"
    if n:
        want = oracle.run_index(x, enc.lengths, enc.total_bits)
        assert np.array_equal(ri.inner[: 2 * want.size].cpu().numpy().view(np.uint16), want)
    before["run_index"] = ri.full.clone()
    # the segment index, likewise
    si = Guarded(max(16, sizes.seg_index_bytes), dev)
    si_status = Guarded(16, dev, fill=0)
    df11.check(df11.df11_build_segment_index(m, si.ptr, si_status.ptr, sh),
               "df11_build_segment_index")
    torch.cuda.synchronize()
    assert int(si_status.inner.cpu().numpy().view(np.uint32)[0]) == 0, "segment index status"
    assert si.margins_intact() and si_status.margins_intact(), \
        "the segment index wrote outside its buffers"
    for k, g in list(bufs.items()) + [("tables", tables), ("run_index", ri)]:
        assert torch.equal(g.full, before[k]), f"the segment index modified its input {k}"
    want = oracle.segment_index(x, enc.lengths, enc.total_bits)
    assert np.array_equal(si.inner[: 4 * want.size].cpu().numpy().view(np.uint32), want)
    before["seg_index"] = si.full.clone()
    for use_index, use_seg in ((False, False), (True, False), (False, True)):
        m.run_index = ri.ptr if use_index else None
        m.seg_index = si.ptr if use_seg else None
        out = Guarded(max(2 * n, 16), dev, fill=0x00)
        status = Guarded(16, dev, fill=0)
        df11.check(df11.df11_decode_block_batch([m], [out.ptr], status.ptr, sh),
                   "df11_decode_block_batch")
        torch.cuda.synchronize()
        assert int(status.inner.cpu().numpy().view(np.uint32)[0]) == 0, "decode status"
        assert out.margins_intact(), "decode wrote outside its output"
        assert status.margins_intact(), "decode wrote outside its status word"
        for k, g in list(bufs.items()) + [("tables", tables), ("run_index", ri), ("seg_index", si)]:
            assert torch.equal(g.full, before[k]), f"decode modified its input {k}"
        got = out.inner[: 2 * n].cpu().numpy().view(np.uint16)
        assert np.array_equal(got, x)
