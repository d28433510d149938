"""Torch-tensor helpers over the DF11 C ABI.

PyTorch provides device memory and streams; every step of compression and
decompression runs in the library (``libdf11_b200.so``): histogram, encode and
decode in its CUDA kernels, codebook and table construction in its C++ host
code.  These helpers only allocate buffers, move the 256-entry histogram and
the small decode tables between host and device, and marshal arguments.

Page: "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70% kích
thước" (vi.news.hada.io/topic?id=20542), sections "Định dạng DFloat11" and
"Giải nén theo từng transformer block".
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

import numpy as np
import torch

from . import (CODEBOOK_BYTES, MAX_CODE_LEN, SEGMENT, TABLE_BITS, DF11Error, check,
               df11_build_codebook, df11_build_segment_index,
               df11_build_codebook_device, df11_build_tables, df11_codebook,
               df11_codebook_from_lengths, df11_decode, df11_decode_block_batch,
               df11_decode_matmul_batch, df11_decode_gemm_batch, df11_decode_host_batch,
               df11_decode_host_scratch_bytes, df11_encode, df11_encode_device_codebook, df11_encoded,
               df11_build_run_index, df11_encoded_sizes, df11_file_bytes, df11_histogram,
               df11_host_matrix, df11_matmul_io,
               df11_matrix, df11_read, df11_sizes, df11_sizes_from_bits, df11_tables_bytes,
               df11_write)


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _as_u16(w: torch.Tensor) -> torch.Tensor:
    if w.dtype == torch.bfloat16:
        w = w.view(torch.int16)
    elif w.dtype not in (torch.int16, torch.uint16):
        raise TypeError(f"expected bfloat16 (or its 16-bit pattern), got {w.dtype}")
    if not w.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    return w.contiguous().reshape(-1)


@dataclass
class DF11Matrix:
    """One compressed matrix resident in device memory."""
    shape: tuple
    n: int
    total_bits: int
    codebook: df11_codebook
    sizes: df11_sizes
    stream: torch.Tensor         # uint8, sizes.stream_alloc
    gaps: torch.Tensor           # uint8, sizes.gaps_alloc
    block_pos: torch.Tensor      # int32 (uint32 bits), sizes.block_pos_alloc / 4
    sign_mantissa: torch.Tensor  # uint8, sizes.sign_mantissa_alloc
    tables: torch.Tensor         # uint8, df11_tables_bytes()
    hist: np.ndarray = field(repr=False, default=None)
    max_block_codes: int = 0     # most codes in one block (0 = unknown)
    run_index: torch.Tensor | None = None  # int16 (uint16 bits), df11_build_run_index
    seg_index: torch.Tensor | None = None  # int32 (uint32 bits), df11_build_segment_index

    def abi(self, use_run_index: bool = True, use_seg_index: bool = True) -> df11_matrix:
        """The C-ABI view.  The decoder takes the segment index when every
        matrix of a launch passes one, else the run index, else neither."""
        ri = self.run_index if (use_run_index and self.run_index is not None) else None
        si = self.seg_index if (use_seg_index and self.seg_index is not None) else None
        return df11_matrix(n=self.n, total_bits=self.total_bits, stream=self.stream.data_ptr(),
                           gaps=self.gaps.data_ptr(), block_pos=self.block_pos.data_ptr(),
                           sign_mantissa=self.sign_mantissa.data_ptr(),
                           tables=self.tables.data_ptr(), min_len=max(1, self.codebook.min_len),
                           max_block_codes=self.max_block_codes,
                           run_index=ri.data_ptr() if ri is not None else None,
                           seg_index=si.data_ptr() if si is not None else None)

    @property
    def stored_bytes(self) -> int:
        """Bytes the format stores (stream, gaps, positions, plane, lengths)."""
        return int(self.sizes.stored_bytes)

    @property
    def ratio(self) -> float:
        return self.stored_bytes / (2 * self.n) if self.n else 0.0

    @property
    def read_bytes(self) -> int:
        """Compressed bytes one decode reads (everything but the lengths)."""
        return int(self.sizes.stored_bytes) - 256

    @property
    def index_bytes(self) -> int:
        """Bytes of the run index (0 without one): read by the indexed decoder."""
        return int(self.sizes.run_index_bytes) if self.run_index is not None else 0

    @property
    def seg_read_bytes(self) -> int:
        """Bytes the segment decoder reads: the stream, the sign/mantissa plane
        and the segment index (not the gaps or block positions)."""
        s = self.sizes
        return int(s.stream_bytes) + int(s.sign_mantissa_bytes) + 4 * (-(-self.n // SEGMENT) + 1)

    def host_arrays(self):
        """Stored arrays copied to the host (for checks and serialisation)."""
        s = self.sizes
        return dict(
            stream=self.stream[: s.stream_bytes].cpu().numpy(),
            gaps=self.gaps[: s.gaps_bytes].cpu().numpy(),
            block_pos=self.block_pos[: s.n_blocks + 1].cpu().numpy().view(np.uint32),
            sign_mantissa=self.sign_mantissa[: s.sign_mantissa_bytes].cpu().numpy(),
            lengths=np.frombuffer(bytes(self.codebook.len), np.uint8).copy(),
        )


def histogram(w: torch.Tensor, stream=None) -> torch.Tensor:
    """256 exponent counts (int64 tensor holding uint64 values) on w's device."""
    u = _as_u16(w)
    h = torch.empty(256, dtype=torch.int64, device=u.device)
    with torch.cuda.device(u.device):
        check(df11_histogram(u.data_ptr(), u.numel(), h.data_ptr(), _stream_handle(stream)),
              "df11_histogram")
    return h


def build_tables(cb: df11_codebook, device) -> torch.Tensor:
    nb = df11_tables_bytes()
    host = np.zeros(nb, np.uint8)
    check(df11_build_tables(cb, host.ctypes.data, nb), "df11_build_tables")
    return torch.from_numpy(host).to(device)


def alloc_encoded(sizes: df11_sizes, device):
    return dict(
        stream=torch.empty(sizes.stream_alloc, dtype=torch.uint8, device=device),
        gaps=torch.empty(sizes.gaps_alloc, dtype=torch.uint8, device=device),
        block_pos=torch.empty(sizes.block_pos_alloc // 4, dtype=torch.int32, device=device),
        sign_mantissa=torch.empty(sizes.sign_mantissa_alloc, dtype=torch.uint8, device=device),
    )


DEFAULT_CAP = TABLE_BITS


def _run_index_for(n: int, total_bits: int, codebook: df11_codebook, sizes: df11_sizes, bufs,
                   tables: torch.Tensor, status_ptr: int, sh: int, dev) -> torch.Tensor | None:
    """Enqueue df11_build_run_index and df11_build_segment_index for freshly
    encoded (or uploaded) buffers; returns the two index tensors (None for an
    empty matrix, and no segment index for a stream of 2^32 bits or more).
    Errors land in the device status word at status_ptr."""
    if n == 0:
        return None, None
    ri = torch.empty(max(16, int(sizes.run_index_bytes)) // 2, dtype=torch.int16, device=dev)
    si = (torch.empty(int(sizes.seg_index_bytes) // 4, dtype=torch.int32, device=dev)
          if total_bits < (1 << 32) else None)
    m = df11_matrix(n=n, total_bits=total_bits, stream=bufs["stream"].data_ptr(),
                    gaps=bufs["gaps"].data_ptr(), block_pos=bufs["block_pos"].data_ptr(),
                    sign_mantissa=bufs["sign_mantissa"].data_ptr(), tables=tables.data_ptr(),
                    min_len=max(1, codebook.min_len), max_block_codes=0, run_index=None)
    with torch.cuda.device(dev):
        check(df11_build_run_index(m, ri.data_ptr(), status_ptr, sh), "df11_build_run_index")
        if si is not None:
            check(df11_build_segment_index(m, si.data_ptr(), status_ptr, sh),
                  "df11_build_segment_index")
    return ri, si


def compress(w: torch.Tensor, cap: int = DEFAULT_CAP, codebook: df11_codebook | None = None,
             stream=None, check_status: bool = True, run_index: bool = True) -> DF11Matrix:
    """BF16 tensor on a CUDA device -> DF11Matrix (GPU histogram, host
    codebook, GPU encode, and by default the run index the decoder uses to
    place every thread's outputs).

    cap is the code-length limit.  The default (11, the decode table's
    reach) lets every code decode on the fast path; for the weight
    distributions measured here it costs about 0.2% more exponent bits
    (0.06% of the compressed size) than the 32-bit limit of the format,
    which remains fully supported (cap=32)."""
    u = _as_u16(w)
    dev = u.device
    sh = _stream_handle(stream)
    h = histogram(u, stream)
    hist = h.cpu().numpy().view(np.uint64).copy()
    if codebook is None:
        st, codebook = df11_build_codebook(hist, cap)
        check(st, "df11_build_codebook")
    st, sizes = df11_encoded_sizes(codebook, hist, u.numel())
    check(st, "df11_encoded_sizes")
    bufs = alloc_encoded(sizes, dev)
    tables = build_tables(codebook, dev)
    ws = torch.empty(max(16, sizes.workspace_bytes), dtype=torch.uint8, device=dev)
    status = torch.zeros(2, dtype=torch.int32, device=dev)  # [status, most codes per block]
    out = df11_encoded(stream=bufs["stream"].data_ptr(), gaps=bufs["gaps"].data_ptr(),
                       block_pos=bufs["block_pos"].data_ptr(),
                       sign_mantissa=bufs["sign_mantissa"].data_ptr(),
                       block_max=status.data_ptr() + 4)
    with torch.cuda.device(dev):
        check(df11_encode(u.data_ptr(), u.numel(), codebook, sizes.total_bits, out,
                          ws.data_ptr(), ws.numel(), status.data_ptr(), sh), "df11_encode")
    ri, si = (_run_index_for(u.numel(), int(sizes.total_bits), codebook, sizes, bufs, tables,
                             status.data_ptr(), sh, dev) if run_index else (None, None))
    st_host = status.cpu().numpy()
    if check_status and int(st_host[0]):
        raise DF11Error(int(st_host[0]), "df11_encode (device)")
    return DF11Matrix(shape=tuple(w.shape), n=u.numel(), total_bits=int(sizes.total_bits),
                      codebook=codebook, sizes=sizes, tables=tables, hist=hist,
                      max_block_codes=int(st_host[1]), run_index=ri, seg_index=si, **bufs)


def compress_block(ws, cap: int = DEFAULT_CAP, stream=None,
                   check_status: bool = True, run_index: bool = True) -> list[DF11Matrix]:
    """Compress several BF16 tensors (e.g. the matrices of a transformer block
    or a whole model) with two host round trips in all: every histogram is
    computed on the device, copied to the host at once, the codebooks and
    decode tables are built on the host, and every encode is enqueued
    before the status words come back in one copy.  The result is the same,
    array for array, as compress() of each tensor."""
    if not ws:
        return []
    us = [_as_u16(w) for w in ws]
    dev = us[0].device
    sh = _stream_handle(stream)
    hists = torch.empty(len(us), 256, dtype=torch.int64, device=dev)
    with torch.cuda.device(dev):
        for i, u in enumerate(us):
            check(df11_histogram(u.data_ptr(), u.numel(), hists[i].data_ptr(), sh), "df11_histogram")
    h_all = hists.cpu().numpy().view(np.uint64).copy()  # round trip 1
    # codebooks, sizes and decode tables on the host; the tables go up in
    # one copy (the device is idle here: nothing is enqueued yet)
    cbs, sizes_l = [], []
    nt = df11_tables_bytes()
    tables_host = np.zeros((len(us), nt), np.uint8)
    for i, u in enumerate(us):
        st, cb = df11_build_codebook(h_all[i], cap)
        check(st, "df11_build_codebook")
        st, sizes = df11_encoded_sizes(cb, h_all[i], u.numel())
        check(st, "df11_encoded_sizes")
        check(df11_build_tables(cb, tables_host[i].ctypes.data, nt), "df11_build_tables")
        cbs.append(cb)
        sizes_l.append(sizes)
    tables = torch.from_numpy(tables_host).to(dev)
    ws_bytes = max(16, max(int(sz.workspace_bytes) for sz in sizes_l))
    wsb = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    status = torch.zeros(len(us), 2, dtype=torch.int32, device=dev)  # [status, most codes per block]
    mats_bufs = []
    with torch.cuda.device(dev):
        for i, (u, cb, sizes) in enumerate(zip(us, cbs, sizes_l)):
            bufs = alloc_encoded(sizes, dev)
            out = df11_encoded(stream=bufs["stream"].data_ptr(), gaps=bufs["gaps"].data_ptr(),
                               block_pos=bufs["block_pos"].data_ptr(),
                               sign_mantissa=bufs["sign_mantissa"].data_ptr(),
                               block_max=status[i].data_ptr() + 4)
            check(df11_encode(u.data_ptr(), u.numel(), cb, sizes.total_bits, out, wsb.data_ptr(),
                              wsb.numel(), status[i].data_ptr(), sh), "df11_encode")
            mats_bufs.append(bufs)
    ris = [(_run_index_for(u.numel(), int(sizes.total_bits), cb, sizes, bufs, tables[i],
                           status[i].data_ptr(), sh, dev) if run_index else (None, None))
           for i, (u, cb, sizes, bufs) in enumerate(zip(us, cbs, sizes_l, mats_bufs))]
    st_host = status.cpu().numpy()  # round trip 2
    mats = []
    for i, (w, u) in enumerate(zip(ws, us)):
        if check_status and int(st_host[i, 0]):
            raise DF11Error(int(st_host[i, 0]), f"df11_encode (device), matrix {i}")
        mats.append(DF11Matrix(shape=tuple(w.shape), n=u.numel(),
                               total_bits=int(sizes_l[i].total_bits), codebook=cbs[i],
                               sizes=sizes_l[i], tables=tables[i], hist=h_all[i],
                               max_block_codes=int(st_host[i, 1]), run_index=ris[i][0],
                               seg_index=ris[i][1], **mats_bufs[i]))
    return mats


# one row per matrix of the device compressor's metadata: the codebook, then
# total_bits (8-byte aligned), padded to 16 bytes
_META_ROW = (CODEBOOK_BYTES + 8 + 15) // 16 * 16
_META_BITS = CODEBOOK_BYTES // 8 * 8


def compress_block_device(ws, cap: int = DEFAULT_CAP, stream=None,
                          check_status: bool = True, run_index: bool = True) -> list[DF11Matrix]:
    """compress_block with every step on the device: histograms, codebooks
    and decode tables (df11_build_codebook_device), encodes with the device
    codebooks (df11_encode_device_codebook).  The host only sizes the
    buffers: one copy of every codebook and bit count, and one copy of the
    status words.  The result equals compress_block's, array for array."""
    if not ws:
        return []
    if CODEBOOK_BYTES % 8:
        raise RuntimeError("unexpected df11_codebook size")
    us = [_as_u16(w) for w in ws]
    dev = us[0].device
    sh = _stream_handle(stream)
    k = len(us)
    nt = df11_tables_bytes()
    hists = torch.empty(k, 256, dtype=torch.int64, device=dev)
    meta = torch.zeros(k, _META_ROW, dtype=torch.uint8, device=dev)
    tables = torch.empty(k, nt, dtype=torch.uint8, device=dev)
    status = torch.zeros(k, 4, dtype=torch.int32, device=dev)  # [status, most codes per block, ...]
    with torch.cuda.device(dev):
        for i, u in enumerate(us):
            check(df11_histogram(u.data_ptr(), u.numel(), hists[i].data_ptr(), sh), "df11_histogram")
            check(df11_build_codebook_device(hists[i].data_ptr(), cap, meta[i].data_ptr(),
                                             tables[i].data_ptr(), meta[i].data_ptr() + _META_BITS,
                                             status[i].data_ptr(), sh),
                  "df11_build_codebook_device")
    meta_h = meta.cpu().numpy()                                      # round trip 1
    st_h = status[:, 0].cpu().numpy()
    h_all = hists.cpu().numpy().view(np.uint64)
    cbs, sizes_l = [], []
    for i, u in enumerate(us):
        if int(st_h[i]):
            raise DF11Error(int(st_h[i]), f"df11_build_codebook_device (device), matrix {i}")
        cb = df11_codebook.from_buffer_copy(meta_h[i, :CODEBOOK_BYTES].tobytes())
        bits = int(meta_h[i, _META_BITS:_META_BITS + 8].view(np.uint64)[0])
        st, sizes = df11_sizes_from_bits(u.numel(), bits)
        check(st, "df11_sizes_from_bits")
        cbs.append(cb)
        sizes_l.append(sizes)
    ws_bytes = max(16, max(int(sz.workspace_bytes) for sz in sizes_l))
    wsb = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    mats_bufs = []
    with torch.cuda.device(dev):
        for i, (u, sizes) in enumerate(zip(us, sizes_l)):
            bufs = alloc_encoded(sizes, dev)
            out = df11_encoded(stream=bufs["stream"].data_ptr(), gaps=bufs["gaps"].data_ptr(),
                               block_pos=bufs["block_pos"].data_ptr(),
                               sign_mantissa=bufs["sign_mantissa"].data_ptr(),
                               block_max=status[i].data_ptr() + 4)
            check(df11_encode_device_codebook(u.data_ptr(), u.numel(), meta[i].data_ptr(),
                                              sizes.total_bits, out, wsb.data_ptr(), wsb.numel(),
                                              status[i].data_ptr(), sh),
                  "df11_encode_device_codebook")
            mats_bufs.append(bufs)
    ris = [(_run_index_for(u.numel(), int(sizes.total_bits), cb, sizes, bufs, tables[i],
                           status[i].data_ptr(), sh, dev) if run_index else (None, None))
           for i, (u, cb, sizes, bufs) in enumerate(zip(us, cbs, sizes_l, mats_bufs))]
    st_host = status.cpu().numpy()                                   # round trip 2
    mats = []
    for i, (w, u) in enumerate(zip(ws, us)):
        if check_status and int(st_host[i, 0]):
            raise DF11Error(int(st_host[i, 0]), f"df11_encode_device_codebook (device), matrix {i}")
        mats.append(DF11Matrix(shape=tuple(w.shape), n=u.numel(),
                               total_bits=int(sizes_l[i].total_bits), codebook=cbs[i],
                               sizes=sizes_l[i], tables=tables[i], hist=h_all[i].copy(),
                               max_block_codes=int(st_host[i, 1]), run_index=ris[i][0],
                               seg_index=ris[i][1], **mats_bufs[i]))
    return mats


def decompress(m: DF11Matrix, out: torch.Tensor | None = None, status: torch.Tensor | None = None,
               stream=None, run_index: bool = True, seg_index: bool = True) -> torch.Tensor:
    """Decode one matrix: with its run index when it has one, else with its
    segment index; run_index / seg_index False leave the index out."""
    dev = m.stream.device
    if out is None:
        out = torch.empty(m.shape, dtype=torch.bfloat16, device=dev)
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(df11_decode(m.abi(run_index, seg_index), out.data_ptr(), status.data_ptr(),
                          _stream_handle(stream)), "df11_decode")
    if own_status:
        s = int(status.item())
        if s:
            raise DF11Error(s, "df11_decode (device)")
    return out


def decompress_block(ms, outs=None, status: torch.Tensor | None = None, stream=None,
                     run_index: bool = True, seg_index: bool = True):
    """Decode every matrix of a block in one launch (the indexed decoder when
    every matrix has a run index, else the segment decoder when every matrix
    has a segment index; run_index / seg_index False leave them out)."""
    dev = ms[0].stream.device
    if outs is None:
        outs = [torch.empty(m.shape, dtype=torch.bfloat16, device=dev) for m in ms]
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(df11_decode_block_batch([m.abi(run_index, seg_index) for m in ms],
                                      [o.data_ptr() for o in outs],
                                      status.data_ptr(), _stream_handle(stream)),
              "df11_decode_block_batch")
    if own_status:
        s = int(status.item())
        if s:
            raise DF11Error(s, "df11_decode_block_batch (device)")
    return outs


@dataclass
class HostMatrix:
    """A compressed matrix whose stored arrays sit in page-locked host memory:
    the input of decompress_host (df11_decode_host_batch)."""
    shape: tuple
    n: int
    total_bits: int
    cap: int
    max_block_codes: int
    arrays: dict            # stream, gaps, block_pos, sign_mantissa, lengths: pinned uint8

    @classmethod
    def from_matrix(cls, m: DF11Matrix) -> "HostMatrix":
        arrays = {}
        for k, v in m.host_arrays().items():
            t = torch.empty(v.nbytes, dtype=torch.uint8, pin_memory=True)
            t.copy_(torch.from_numpy(np.ascontiguousarray(v).view(np.uint8)))
            arrays[k] = t
        return cls(tuple(m.shape), m.n, m.total_bits, int(m.codebook.cap),
                   int(m.max_block_codes), arrays)

    @property
    def h2d_bytes(self) -> int:
        """Bytes one decode copies to the device (the four stored arrays)."""
        return sum(self.arrays[k].numel() for k in ("stream", "gaps", "block_pos",
                                                    "sign_mantissa"))

    def abi(self) -> df11_host_matrix:
        hm = df11_host_matrix(n=self.n, total_bits=self.total_bits, cap=self.cap,
                              max_block_codes=self.max_block_codes, ndim=0)
        for k in ("lengths", "gaps", "block_pos", "stream", "sign_mantissa"):
            setattr(hm, k, self.arrays[k].data_ptr())
        return hm


def host_scratch(hms, device) -> torch.Tensor:
    """Device scratch for decompress_host over these matrices."""
    size = df11_decode_host_scratch_bytes([h.abi() for h in hms])
    if size == 0 and hms:
        raise DF11Error(1, "df11_decode_host_scratch_bytes")
    return torch.empty(max(size, 256), dtype=torch.uint8, device=device)


def decompress_host(hms, outs=None, scratch: torch.Tensor | None = None,
                    status: torch.Tensor | None = None, stream=None, device="cuda"):
    """Decode host-resident matrices into page-locked host BF16 tensors:
    copies in, run index, decode and copies out pipelined by the library.
    With a caller's status the call returns with the work queued on stream;
    without one it waits and raises on a device-reported error."""
    if outs is None:
        outs = [torch.empty(h.shape, dtype=torch.bfloat16, pin_memory=True) for h in hms]
    if scratch is None:
        scratch = host_scratch(hms, device)
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device=scratch.device)
    with torch.cuda.device(scratch.device):
        check(df11_decode_host_batch([h.abi() for h in hms], [o.data_ptr() for o in outs],
                                     scratch.data_ptr(), scratch.numel(), status.data_ptr(),
                                     _stream_handle(stream)), "df11_decode_host_batch")
    if own_status:
        (stream if stream is not None else torch.cuda.current_stream(scratch.device)).synchronize()
        s = int(status.item())
        if s:
            raise DF11Error(s, "df11_decode_host_batch (device)")
    return outs


def matmul_block(ms, xs, ys=None, status: torch.Tensor | None = None, stream=None):
    """y_i = x_i W_i^T for every matrix W_i of a block (each of shape
    rows x cols, as compressed), decoded on the fly in one launch: the BF16
    weights never reach device memory.  xs: BF16 tensors of shape
    (batch, cols_i), batch <= MATMUL_MAX_BATCH; ys: FP32 tensors of shape
    (batch, rows_i), zeroed here when not given (the products are added)."""
    dev = ms[0].stream.device
    batch = int(xs[0].shape[0])
    for m, x in zip(ms, xs):
        if len(m.shape) != 2 or x.dtype != torch.bfloat16 or x.shape != (batch, m.shape[1]):
            raise ValueError("matmul_block: x must be BF16 (batch, cols) for a rows x cols matrix")
    xs = [x.contiguous() for x in xs]
    if ys is None:
        ys = [torch.zeros(batch, m.shape[0], dtype=torch.float32, device=dev) for m in ms]
    ios = [df11_matmul_io(rows=m.shape[0], cols=m.shape[1], x=x.data_ptr(), y=y.data_ptr())
           for m, x, y in zip(ms, xs, ys)]
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(df11_decode_matmul_batch([m.abi() for m in ms], ios, batch, status.data_ptr(),
                                       _stream_handle(stream)), "df11_decode_matmul_batch")
    if own_status:
        s = int(status.item())
        if s:
            raise DF11Error(s, "df11_decode_matmul_batch (device)")
    return ys


def gemm_block(ms, xs, ys=None, status: torch.Tensor | None = None, stream=None):
    """y_i = x_i W_i^T for every matrix W_i of a block on the tensor cores
    (df11_decode_gemm_batch): W_i decoded through its segment index into the
    MMA's operand tiles, never written to device memory.  xs: BF16 tensors of
    shape (batch, cols_i) with cols_i a multiple of SEGMENT, any batch; ys:
    FP32 (batch, rows_i), zeroed here when not given (the products are
    added)."""
    dev = ms[0].stream.device
    batch = int(xs[0].shape[0])
    for m, x in zip(ms, xs):
        if len(m.shape) != 2 or x.dtype != torch.bfloat16 or x.shape != (batch, m.shape[1]):
            raise ValueError("gemm_block: x must be BF16 (batch, cols) for a rows x cols matrix")
        if m.seg_index is None:
            raise ValueError("gemm_block: the matrix has no segment index")
    xs = [x.contiguous() for x in xs]
    if ys is None:
        ys = [torch.zeros(batch, m.shape[0], dtype=torch.float32, device=dev) for m in ms]
    ios = [df11_matmul_io(rows=m.shape[0], cols=m.shape[1], x=x.data_ptr(), y=y.data_ptr())
           for m, x, y in zip(ms, xs, ys)]
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(df11_decode_gemm_batch([m.abi() for m in ms], ios, batch, status.data_ptr(),
                                     _stream_handle(stream)), "df11_decode_gemm_batch")
    if own_status:
        s = int(status.item())
        if s:
            raise DF11Error(s, "df11_decode_gemm_batch (device)")
    return ys


def from_host_arrays(shape, n: int, total_bits: int, codebook: df11_codebook, stream, gaps,
                     block_pos, sign_mantissa, device, run_index: bool = True) -> DF11Matrix:
    """Upload stored arrays (e.g. produced elsewhere) into padded device
    buffers ready for decoding."""
    hist = np.zeros(256, np.uint64)
    st, sizes = df11_sizes_from_bits(n, total_bits)
    check(st, "df11_sizes_from_bits")

    def padded(a, size, dtype=np.uint8):
        buf = np.zeros(size // np.dtype(dtype).itemsize, dtype)
        a = np.asarray(a).view(dtype).reshape(-1)
        buf[: a.size] = a
        return torch.from_numpy(buf).to(device)

    bufs = dict(stream=padded(stream, sizes.stream_alloc), gaps=padded(gaps, sizes.gaps_alloc),
                block_pos=padded(np.asarray(block_pos, np.uint32).view(np.int32),
                                 sizes.block_pos_alloc, np.int32),
                sign_mantissa=padded(sign_mantissa, sizes.sign_mantissa_alloc))
    tables = build_tables(codebook, device)
    ri = si = None
    if run_index and n:
        # the index of data from elsewhere is built here, on the device; a
        # stream that does not match its positions is reported
        dev = bufs["stream"].device
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        ri, si = _run_index_for(n, total_bits, codebook, sizes, bufs, tables, status.data_ptr(),
                                _stream_handle(None), dev)
        st = int(status.item())
        if st:
            raise DF11Error(st, "df11_build_run_index / df11_build_segment_index (device)")
    return DF11Matrix(shape=tuple(shape), n=n, total_bits=total_bits, codebook=codebook,
                      sizes=sizes, tables=tables, hist=hist, run_index=ri, seg_index=si, **bufs)


def serialize(m: DF11Matrix) -> np.ndarray:
    """The matrix in the .df11 container (include/df11.h), as a uint8 array."""
    h = m.host_arrays()
    arrs = {k: np.ascontiguousarray(v) for k, v in h.items()}
    hm = df11_host_matrix(n=m.n, total_bits=m.total_bits, cap=int(m.codebook.cap),
                          max_block_codes=int(m.max_block_codes), ndim=len(m.shape))
    if len(m.shape) > 4:
        raise ValueError("serialize: at most 4 dimensions")
    for i, d in enumerate(m.shape):
        hm.shape[i] = int(d)
    hm.lengths = arrs["lengths"].ctypes.data
    hm.gaps = arrs["gaps"].ctypes.data
    hm.block_pos = arrs["block_pos"].ctypes.data
    hm.stream = arrs["stream"].ctypes.data
    hm.sign_mantissa = arrs["sign_mantissa"].ctypes.data
    size = df11_file_bytes(m.n, m.total_bits)
    buf = np.empty(size, np.uint8)
    st, written = df11_write(hm, buf.ctypes.data, size)
    check(st, "df11_write")
    assert written == size
    return buf


def deserialize(data, device) -> DF11Matrix:
    """A matrix read from the .df11 container (bytes or a uint8 array), checked
    (magic, sizes, CRC-32, metadata) by the library and uploaded to device."""
    buf = np.frombuffer(data, np.uint8) if not isinstance(data, np.ndarray) else data
    buf = np.ascontiguousarray(buf, np.uint8)
    st, hm = df11_read(buf.ctypes.data, buf.size)
    check(st, "df11_read")
    base = buf.ctypes.data
    st, sizes = df11_sizes_from_bits(hm.n, hm.total_bits)
    check(st, "df11_sizes_from_bits")

    def view(ptr, nbytes):
        off = int(ptr) - base
        return buf[off:off + int(nbytes)]

    lengths = view(hm.lengths, 256)
    st, cb = df11_codebook_from_lengths(lengths.ctypes.data, int(hm.cap) or MAX_CODE_LEN)
    check(st, "df11_codebook_from_lengths")
    shape = tuple(int(hm.shape[i]) for i in range(hm.ndim)) if hm.ndim else (int(hm.n),)
    m = from_host_arrays(shape, int(hm.n), int(hm.total_bits), cb,
                         view(hm.stream, sizes.stream_bytes), view(hm.gaps, sizes.gaps_bytes),
                         view(hm.block_pos, sizes.block_pos_bytes).view(np.uint32),
                         view(hm.sign_mantissa, sizes.sign_mantissa_bytes), device)
    m.max_block_codes = int(hm.max_block_codes)
    return m


def save(path: str, m: DF11Matrix) -> int:
    """Write the matrix to a .df11 file; returns the bytes written."""
    buf = serialize(m)
    with open(path, "wb") as f:
        f.write(buf.tobytes())
    return int(buf.size)


def load(path: str, device="cuda") -> DF11Matrix:
    """Read a .df11 file into device buffers ready for decoding."""
    with open(path, "rb") as f:
        data = f.read()
    return deserialize(data, device)


def codebook_from_lengths(lengths, codes) -> df11_codebook:
    cb = df11_codebook()
    ln = [int(x) for x in lengths]
    for i in range(256):
        cb.len[i] = ln[i]
        cb.code[i] = int(codes[i])
    nz = [x for x in ln if x]
    cb.max_len = max(nz) if nz else 0
    cb.min_len = min(nz) if nz else 0
    cb.n_symbols = len(nz)
    cb.cap = MAX_CODE_LEN
    return cb


__all__ = ["DF11Matrix", "histogram", "compress", "decompress", "decompress_block",
           "build_tables", "alloc_encoded", "from_host_arrays", "codebook_from_lengths",
           "serialize", "deserialize", "save", "load", "ctypes"]
