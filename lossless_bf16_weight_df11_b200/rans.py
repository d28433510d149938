"""Torch-tensor helpers for the rANS variant of the exponent coding
(``include/df11_rans.h``), the comparison codec for DF11's Huffman code.

As in ``codec``: PyTorch allocates, the library computes.  The histogram,
both encoding passes and the decode run in the library's CUDA kernels; the
frequencies and tables are built by its host code.  Per matrix the host sees
the 256-entry histogram and the stream size (one 4-byte copy);
``compress_block`` batches those round trips over many matrices.

Page: "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70% kích
thước" (vi.news.hada.io/topic?id=20542); its Hacker News discussion names rANS
as the alternative to the Huffman exponent code.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from . import (RANS_TABLES_BYTES, DF11Error, check, df11_histogram, df11_rans_build_tables,
               df11_rans_decode_batch, df11_rans_encode, df11_rans_encode_sizes, df11_rans_freqs,
               df11_rans_matrix, df11_rans_units)
from .codec import _as_u16, _stream_handle


@dataclass
class RansMatrix:
    """One rANS-coded matrix resident in device memory."""
    shape: tuple
    n: int
    freq: np.ndarray             # uint32[256], sum 4096 (all zero for n = 0)
    stream_bytes: int            # off16[U] * 16
    stream: torch.Tensor         # uint8, max(16, stream_bytes)
    off16: torch.Tensor          # int32 (uint32 bits), U + 1
    sign_mantissa: torch.Tensor  # uint8, n rounded up to 16
    tables: torch.Tensor         # uint8, RANS_TABLES_BYTES
    hist: np.ndarray = field(repr=False, default=None)

    @property
    def units(self) -> int:
        return int(self.off16.numel()) - 1

    def abi(self) -> df11_rans_matrix:
        return df11_rans_matrix(n=self.n, stream=self.stream.data_ptr(),
                                off16=self.off16.data_ptr(),
                                sign_mantissa=self.sign_mantissa.data_ptr(),
                                tables=self.tables.data_ptr())

    @property
    def stored_bytes(self) -> int:
        """Stream, unit offsets, sign/mantissa plane and 256 16-bit frequencies."""
        return self.stream_bytes + 4 * (self.units + 1) + self.n + 512

    @property
    def read_bytes(self) -> int:
        """Compressed bytes one decode reads (everything but the frequencies;
        the 16 KiB slot table is read once per CTA from L2)."""
        return self.stored_bytes - 512

    @property
    def ratio(self) -> float:
        return self.stored_bytes / (2 * self.n) if self.n else 0.0

    def host_arrays(self):
        return dict(stream=self.stream[: self.stream_bytes].cpu().numpy(),
                    off16=self.off16.cpu().numpy().view(np.uint32),
                    sign_mantissa=self.sign_mantissa[: self.n].cpu().numpy(),
                    freq=self.freq.copy())


def _host_tables(freq: np.ndarray) -> np.ndarray:
    host = np.zeros(RANS_TABLES_BYTES, np.uint8)
    check(df11_rans_build_tables(freq, host.ctypes.data, host.size), "df11_rans_build_tables")
    return host


def compress_block(ws, freqs=None, stream=None, check_status: bool = True) -> list[RansMatrix]:
    """Compress BF16 tensors with three host round trips in all: the
    histograms, the stream sizes, and the status words.  freqs: optional
    per-tensor frequency arrays to use instead of the histograms' own."""
    if not ws:
        return []
    us = [_as_u16(w) for w in ws]
    dev = us[0].device
    sh = _stream_handle(stream)
    hists = torch.empty(len(us), 256, dtype=torch.int64, device=dev)
    with torch.cuda.device(dev):
        for i, u in enumerate(us):
            check(df11_histogram(u.data_ptr(), u.numel(), hists[i].data_ptr(), sh), "df11_histogram")
    h_all = hists.cpu().numpy().view(np.uint64).copy()          # round trip 1
    fs = []
    for i in range(len(us)):
        if freqs is not None and freqs[i] is not None:
            fs.append(np.ascontiguousarray(freqs[i], np.uint32))
        else:
            st, f = df11_rans_freqs(h_all[i])
            check(st, "df11_rans_freqs")
            fs.append(np.array(f, np.uint32))
    tables = torch.from_numpy(np.stack([_host_tables(f) for f in fs])).to(dev)
    units = [df11_rans_units(u.numel()) for u in us]
    unit_words = [torch.empty(max(1, U), dtype=torch.int32, device=dev) for U in units]
    off16 = [torch.empty(U + 1, dtype=torch.int32, device=dev) for U in units]
    status = torch.zeros(len(us), 4, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        for i, u in enumerate(us):
            check(df11_rans_encode_sizes(u.data_ptr(), u.numel(), tables[i].data_ptr(),
                                         unit_words[i].data_ptr(), off16[i].data_ptr(),
                                         status[i].data_ptr(), sh), "df11_rans_encode_sizes")
    ends = torch.stack([o[-1] for o in off16]).cpu().numpy().view(np.uint32)  # round trip 2
    mats = []
    with torch.cuda.device(dev):
        for i, (w, u) in enumerate(zip(ws, us)):
            sb = int(ends[i]) * 16
            s_buf = torch.empty(max(16, sb), dtype=torch.uint8, device=dev)
            sm = torch.empty(max(16, (u.numel() + 15) // 16 * 16), dtype=torch.uint8, device=dev)
            check(df11_rans_encode(u.data_ptr(), u.numel(), tables[i].data_ptr(),
                                   unit_words[i].data_ptr(), off16[i].data_ptr(), s_buf.data_ptr(),
                                   sm.data_ptr(), status[i].data_ptr(), sh), "df11_rans_encode")
            mats.append(RansMatrix(shape=tuple(w.shape), n=u.numel(), freq=fs[i], stream_bytes=sb,
                                   stream=s_buf, off16=off16[i], sign_mantissa=sm,
                                   tables=tables[i], hist=h_all[i]))
    st_host = status[:, 0].cpu().numpy()                        # round trip 3
    if check_status:
        for i, s in enumerate(st_host):
            if int(s):
                raise DF11Error(int(s), f"rANS encode (device), matrix {i}")
    return mats


def compress(w: torch.Tensor, freq=None, stream=None, check_status: bool = True) -> RansMatrix:
    return compress_block([w], None if freq is None else [freq], stream, check_status)[0]


def decompress_block(ms, outs=None, status: torch.Tensor | None = None, stream=None):
    """Decode every matrix (one launch per 32)."""
    dev = ms[0].stream.device
    if outs is None:
        outs = [torch.empty(m.shape, dtype=torch.bfloat16, device=dev) for m in ms]
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        check(df11_rans_decode_batch([m.abi() for m in ms], [o.data_ptr() for o in outs],
                                     status.data_ptr(), _stream_handle(stream)),
              "df11_rans_decode_batch")
    if own_status:
        s = int(status.item())
        if s:
            raise DF11Error(s, "df11_rans_decode_batch (device)")
    return outs


def decompress(m: RansMatrix, out: torch.Tensor | None = None, status=None, stream=None):
    return decompress_block([m], None if out is None else [out], status, stream)[0]


def from_host_arrays(shape, n: int, freq, stream, off16, sign_mantissa, device) -> RansMatrix:
    """Upload stored arrays (e.g. the oracle's) into device buffers."""
    freq = np.ascontiguousarray(freq, np.uint32)
    stream = np.ascontiguousarray(stream, np.uint8)
    s_buf = np.zeros(max(16, stream.size), np.uint8)
    s_buf[: stream.size] = stream
    sm = np.zeros(max(16, (n + 15) // 16 * 16), np.uint8)
    sm[:n] = np.asarray(sign_mantissa, np.uint8)[:n]
    return RansMatrix(shape=tuple(shape), n=n, freq=freq, stream_bytes=stream.size,
                      stream=torch.from_numpy(s_buf).to(device),
                      off16=torch.from_numpy(np.ascontiguousarray(off16, np.uint32).view(np.int32)
                                             .copy()).to(device),
                      sign_mantissa=torch.from_numpy(sm).to(device),
                      tables=torch.from_numpy(_host_tables(freq)).to(device))


__all__ = ["RansMatrix", "compress", "compress_block", "decompress", "decompress_block",
           "from_host_arrays"]
