"""Plain CPU oracle for the DF11 lossless BF16 codec -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline arm of
``bench.py`` may import this package.  The product library never imports,
links or calls it, and it shares no code with the CUDA path: the arithmetic
lives in ``df11_oracle.c`` (plain C, single-threaded, bit-serial) and this
module only marshals numpy arrays to it.

Method source: the page "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM
xuống còn 70% kích thước" (vi.news.hada.io/topic?id=20542), sections "Định dạng
DFloat11" (format), "Dư địa nén còn lại trong exponent của BFloat16" (exponent
statistics) and "Kernel GPU hai giai đoạn và metadata bổ trợ" (chunks, gaps,
block output positions).  The readings the page leaves open are listed at the
top of ``df11_oracle.c``; those of the rANS comparison variant (which the
page's discussion only names) above its section there.

Parity status: every DF11 entry point is pinned by ``tests/test_oracle_pins.py``
and every rANS entry point by ``tests/test_oracle_rans.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "df11_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libdf11_oracle.so")

CHUNK_BITS = 64
BLOCK_CHUNKS = 256
GAP_BITS = 5
MAX_CAP = 32

OK, ERR_ARG, ERR_SYMBOL, ERR_CORRUPT = 0, 1, 2, 3

_lock = threading.Lock()
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc -O2 (no threads, no intrinsics)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=c99", "-Wall", "-shared", "-fPIC", src, "-o", tmp, "-lm"],
                   check=True)
    os.replace(tmp, out)
    return out


_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u64p = ctypes.POINTER(ctypes.c_uint64)


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    c_u64, c_int = ctypes.c_uint64, ctypes.c_int
    sig = {
        "oracle_split": (None, [_u16p, c_u64, _u8p, _u8p]),
        "oracle_merge": (None, [_u8p, _u8p, c_u64, _u16p]),
        "oracle_histogram": (None, [_u8p, c_u64, _u64p]),
        "oracle_entropy": (ctypes.c_double, [_u64p]),
        "oracle_huffman_lengths": (c_int, [_u64p, _u8p]),
        "oracle_package_merge": (c_int, [_u64p, c_int, _u8p]),
        "oracle_normalize_lengths": (None, [_u64p, _u8p]),
        "oracle_canonical_codes": (None, [_u8p, _u32p]),
        "oracle_codebook": (c_int, [_u64p, c_int, _u8p, _u32p]),
        "oracle_total_bits": (c_int, [_u8p, c_u64, _u8p, _u64p]),
        "oracle_encode": (c_int, [_u8p, c_u64, _u8p, _u32p, c_u64, _u8p, _u8p, _u32p]),
        "oracle_pack_gaps": (None, [_u8p, c_u64, _u8p]),
        "oracle_run_index": (c_int, [_u8p, c_u64, _u8p, c_u64, ctypes.POINTER(ctypes.c_uint16)]),
        "oracle_segment_index": (c_int, [_u8p, c_u64, _u8p, c_u64, _u32p]),
        "oracle_unpack_gaps": (None, [_u8p, c_u64, _u8p]),
        "oracle_decode_serial": (c_int, [_u8p, c_u64, c_u64, _u8p, _u32p, _u8p]),
        "oracle_decode_chunked": (c_int, [_u8p, _u8p, _u32p, c_u64, c_u64, _u8p, _u32p, _u8p]),
        "oracle_rans_freqs": (c_int, [_u64p, _u32p]),
        "oracle_rans_bound": (c_u64, [c_u64]),
        "oracle_rans_encode": (c_int, [_u8p, c_u64, _u32p, _u8p, c_u64, _u32p, _u64p]),
        "oracle_rans_decode": (c_int, [_u8p, _u32p, c_u64, _u32p, _u8p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load(path: str | None = None) -> ctypes.CDLL:
    """Build (if needed) and load the oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _p(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


# ---------------------------------------------------------------- steps


def split(w: np.ndarray, lib=None):
    """BF16 words (uint16) -> (exponent bytes, sign+mantissa bytes)."""
    lib = lib or load()
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    e = np.empty(w.size, np.uint8)
    sm = np.empty(w.size, np.uint8)
    lib.oracle_split(_p(w, _u16p), w.size, _p(e, _u8p), _p(sm, _u8p))
    return e, sm


def merge(e: np.ndarray, sm: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    w = np.empty(e.size, np.uint16)
    lib.oracle_merge(_p(e, _u8p), _p(sm, _u8p), e.size, _p(w, _u16p))
    return w


def histogram(e: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    e = np.ascontiguousarray(e, dtype=np.uint8).reshape(-1)
    h = np.zeros(256, np.uint64)
    lib.oracle_histogram(_p(e, _u8p), e.size, _p(h, _u64p))
    return h


def entropy(hist: np.ndarray, lib=None) -> float:
    lib = lib or load()
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    return float(lib.oracle_entropy(_p(h, _u64p)))


def huffman_lengths(hist: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    ln = np.zeros(256, np.uint8)
    lib.oracle_huffman_lengths(_p(h, _u64p), _p(ln, _u8p))
    return ln


def package_merge(hist: np.ndarray, cap: int, lib=None) -> np.ndarray:
    lib = lib or load()
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    ln = np.zeros(256, np.uint8)
    r = lib.oracle_package_merge(_p(h, _u64p), cap, _p(ln, _u8p))
    if r < 0:
        raise ValueError(f"cap {cap} cannot hold {int((h > 0).sum())} symbols")
    return ln


def normalize_lengths(hist: np.ndarray, lengths: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    ln = np.array(lengths, dtype=np.uint8, copy=True)
    lib.oracle_normalize_lengths(_p(h, _u64p), _p(ln, _u8p))
    return ln


def canonical_codes(lengths: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    ln = np.ascontiguousarray(lengths, dtype=np.uint8)
    code = np.zeros(256, np.uint32)
    lib.oracle_canonical_codes(_p(ln, _u8p), _p(code, _u32p))
    return code


def codebook(hist: np.ndarray, cap: int = MAX_CAP, lib=None):
    """Histogram -> (code lengths uint8[256], canonical codes uint32[256])."""
    lib = lib or load()
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    ln = np.zeros(256, np.uint8)
    code = np.zeros(256, np.uint32)
    r = lib.oracle_codebook(_p(h, _u64p), cap, _p(ln, _u8p), _p(code, _u32p))
    if r < 0:
        raise ValueError("cap too small for the alphabet")
    return ln, code


def pack_gaps(gaps: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or load()
    g = np.ascontiguousarray(gaps, dtype=np.uint8)
    out = np.zeros((GAP_BITS * g.size + 7) // 8, np.uint8)
    lib.oracle_pack_gaps(_p(g, _u8p), g.size, _p(out, _u8p))
    return out


def unpack_gaps(packed: np.ndarray, chunks: int, lib=None) -> np.ndarray:
    lib = lib or load()
    pk = np.ascontiguousarray(packed, dtype=np.uint8)
    assert pk.size * 8 >= GAP_BITS * chunks
    g = np.zeros(chunks, np.uint8)
    lib.oracle_unpack_gaps(_p(pk, _u8p), chunks, _p(g, _u8p))
    return g


@dataclass
class Encoded:
    """Everything the format stores for one matrix (plus the exponents)."""
    n: int
    hist: np.ndarray          # uint64[256]
    lengths: np.ndarray       # uint8[256]
    codes: np.ndarray         # uint32[256]
    total_bits: int
    stream: np.ndarray        # uint8[8*C]   EncodedExponent
    gaps: np.ndarray          # uint8[C]     one gap per chunk, unpacked
    gaps_packed: np.ndarray   # uint8[ceil(5C/8)]
    block_pos: np.ndarray     # uint32[B+1]
    sign_mantissa: np.ndarray  # uint8[n]    PackedSignMantissa

    @property
    def n_chunks(self) -> int:
        return (self.total_bits + CHUNK_BITS - 1) // CHUNK_BITS

    @property
    def n_blocks(self) -> int:
        return (self.n_chunks + BLOCK_CHUNKS - 1) // BLOCK_CHUNKS


def encode(w: np.ndarray, cap: int = MAX_CAP, lengths=None, codes=None, lib=None) -> Encoded:
    """Full compressor: split, histogram, codebook, bit-serial encode."""
    lib = lib or load()
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    n = w.size
    e, sm = split(w, lib)
    h = histogram(e, lib)
    if lengths is None:
        lengths, codes = codebook(h, cap, lib)
    lengths = np.ascontiguousarray(lengths, dtype=np.uint8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    tb = ctypes.c_uint64(0)
    r = lib.oracle_total_bits(_p(e, _u8p), n, _p(lengths, _u8p), ctypes.byref(tb))
    if r != OK:
        raise ValueError("a value to encode has no code")
    total_bits = int(tb.value)
    chunks = (total_bits + CHUNK_BITS - 1) // CHUNK_BITS
    blocks = (chunks + BLOCK_CHUNKS - 1) // BLOCK_CHUNKS
    stream = np.zeros(8 * chunks, np.uint8)
    gaps = np.zeros(chunks, np.uint8)
    pos = np.zeros(blocks + 1, np.uint32)
    r = lib.oracle_encode(_p(e, _u8p), n, _p(lengths, _u8p), _p(codes, _u32p), total_bits,
                          _p(stream, _u8p), _p(gaps, _u8p), _p(pos, _u32p))
    if r != OK:
        raise ValueError(f"oracle_encode failed with {r}")
    return Encoded(n=n, hist=h, lengths=lengths, codes=codes, total_bits=total_bits,
                   stream=stream, gaps=gaps, gaps_packed=pack_gaps(gaps, lib), block_pos=pos,
                   sign_mantissa=sm)


def run_index(w: np.ndarray, lengths, total_bits: int, lib=None) -> np.ndarray:
    """R12: for each 128-bit run of each 256-chunk block, the number of codes
    that start in the block before the run (uint16, 128 per block)."""
    lib = lib or load()
    e, _ = split(w, lib)
    chunks = (total_bits + CHUNK_BITS - 1) // CHUNK_BITS
    blocks = (chunks + BLOCK_CHUNKS - 1) // BLOCK_CHUNKS
    out = np.zeros(blocks * (BLOCK_CHUNKS // 2), np.uint16)
    r = lib.oracle_run_index(_p(e, _u8p), e.size, _p(np.ascontiguousarray(lengths, np.uint8), _u8p),
                             total_bits, _p(out, ctypes.POINTER(ctypes.c_uint16)))
    if r != OK:
        raise ValueError(f"oracle_run_index failed with {r}")
    return out


SEGMENT = 64  # outputs per segment of the segment index


def segment_index(w: np.ndarray, lengths, total_bits: int, lib=None) -> np.ndarray:
    """R13: the stream bit at which the code of value 64j starts, for
    j < ceil(n/64), then total_bits (uint32, ceil(n/64) + 1 entries)."""
    lib = lib or load()
    e, _ = split(w, lib)
    out = np.zeros((e.size + SEGMENT - 1) // SEGMENT + 1, np.uint32)
    r = lib.oracle_segment_index(_p(e, _u8p), e.size,
                                 _p(np.ascontiguousarray(lengths, np.uint8), _u8p), total_bits,
                                 _p(out, _u32p))
    if r != OK:
        raise ValueError(f"oracle_segment_index failed with {r}")
    return out


def decode_serial_exponents(stream, total_bits: int, n: int, lengths, codes, lib=None) -> np.ndarray:
    lib = lib or load()
    s = np.ascontiguousarray(stream, dtype=np.uint8)
    assert s.size * 8 >= total_bits
    e = np.zeros(n, np.uint8)
    r = lib.oracle_decode_serial(_p(s, _u8p), total_bits, n,
                                 _p(np.ascontiguousarray(lengths, np.uint8), _u8p),
                                 _p(np.ascontiguousarray(codes, np.uint32), _u32p), _p(e, _u8p))
    if r != OK:
        raise ValueError("stream is corrupt")
    return e


def decode_chunked_exponents(stream, gaps, block_pos, total_bits: int, n: int, lengths, codes,
                             lib=None) -> np.ndarray:
    lib = lib or load()
    s = np.ascontiguousarray(stream, dtype=np.uint8)
    g = np.ascontiguousarray(gaps, dtype=np.uint8)
    pos = np.ascontiguousarray(block_pos, dtype=np.uint32)
    chunks = (total_bits + CHUNK_BITS - 1) // CHUNK_BITS
    blocks = (chunks + BLOCK_CHUNKS - 1) // BLOCK_CHUNKS
    assert s.size * 8 >= total_bits and g.size >= chunks and pos.size >= blocks + 1
    e = np.zeros(n, np.uint8)
    r = lib.oracle_decode_chunked(_p(s, _u8p), _p(g, _u8p), _p(pos, _u32p), total_bits, n,
                                  _p(np.ascontiguousarray(lengths, np.uint8), _u8p),
                                  _p(np.ascontiguousarray(codes, np.uint32), _u32p), _p(e, _u8p))
    if r != OK:
        raise ValueError("stream or metadata is corrupt")
    return e


def decode(enc: Encoded, chunked: bool = False, lib=None) -> np.ndarray:
    """Encoded matrix -> BF16 words (uint16), bit-serial."""
    lib = lib or load()
    if chunked:
        e = decode_chunked_exponents(enc.stream, enc.gaps, enc.block_pos, enc.total_bits, enc.n,
                                     enc.lengths, enc.codes, lib)
    else:
        e = decode_serial_exponents(enc.stream, enc.total_bits, enc.n, enc.lengths, enc.codes, lib)
    return merge(e, enc.sign_mantissa, lib)


def stored_bytes(enc: Encoded) -> int:
    """Bytes the format stores: stream, packed gaps, block positions,
    sign+mantissa plane and the 256 code lengths."""
    return (enc.stream.size + enc.gaps_packed.size + 4 * enc.block_pos.size
            + enc.sign_mantissa.size + 256)


# ---- rANS variant of the exponent coding (comparison codec; the format's
# readings Q1-Q5 are listed in df11_oracle.c)

RANS_M = 4096
RANS_L = 1 << 16
RANS_LANES = 32
RANS_STEPS = 512
RANS_SEG_STEPS = 64
RANS_SEGS = RANS_STEPS // RANS_SEG_STEPS
RANS_UNIT = RANS_LANES * RANS_STEPS
RANS_HEADER = 4 * RANS_LANES + 2 * RANS_SEGS


def rans_freqs(hist: np.ndarray, lib=None) -> np.ndarray:
    """Frequencies out of 4096 for a 256-bin histogram (Q1)."""
    lib = lib or load()
    h = np.ascontiguousarray(hist, dtype=np.uint64)
    f = np.zeros(256, np.uint32)
    if lib.oracle_rans_freqs(_p(h, _u64p), _p(f, _u32p)) != OK:
        raise ValueError("rans_freqs failed")
    return f


@dataclass
class RansEncoded:
    n: int
    hist: np.ndarray          # uint64[256]
    freq: np.ndarray          # uint32[256], sum 4096 (or all zero for n = 0)
    stream: np.ndarray        # uint8[bytes]: the units back to back
    off16: np.ndarray         # uint32[U+1]: unit starts in 16-byte units
    sign_mantissa: np.ndarray  # uint8[n]

    @property
    def units(self) -> int:
        return (self.n + RANS_UNIT - 1) // RANS_UNIT


def rans_encode(w: np.ndarray, freq=None, lib=None) -> RansEncoded:
    """Split, histogram, frequencies (Q1) and the interleaved encode (Q2-Q4)."""
    lib = lib or load()
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    n = w.size
    e, sm = split(w, lib)
    h = histogram(e, lib)
    f = rans_freqs(h, lib) if freq is None else np.ascontiguousarray(freq, np.uint32)
    units = (n + RANS_UNIT - 1) // RANS_UNIT
    cap = int(lib.oracle_rans_bound(n))
    stream = np.zeros(max(cap, 16), np.uint8)
    off16 = np.zeros(units + 1, np.uint32)
    nbytes = ctypes.c_uint64(0)
    r = lib.oracle_rans_encode(_p(e, _u8p), n, _p(f, _u32p), _p(stream, _u8p), stream.size,
                               _p(off16, _u32p), ctypes.byref(nbytes))
    if r != OK:
        raise ValueError(f"oracle_rans_encode failed with {r}")
    return RansEncoded(n=n, hist=h, freq=f, stream=stream[: int(nbytes.value)].copy(),
                       off16=off16, sign_mantissa=sm)


def rans_decode(enc: RansEncoded, lib=None) -> np.ndarray:
    """Definition-level decode (linear symbol search per value) -> BF16 words."""
    lib = lib or load()
    e = np.zeros(enc.n, np.uint8)
    s = np.ascontiguousarray(enc.stream, np.uint8)
    if s.size == 0:
        s = np.zeros(16, np.uint8)
    r = lib.oracle_rans_decode(_p(s, _u8p), _p(np.ascontiguousarray(enc.off16, np.uint32), _u32p),
                               enc.n, _p(np.ascontiguousarray(enc.freq, np.uint32), _u32p),
                               _p(e, _u8p))
    if r != OK:
        raise ValueError("rANS stream is corrupt")
    return merge(e, enc.sign_mantissa, lib)


def rans_stored_bytes(enc: RansEncoded) -> int:
    """Bytes the rANS variant stores: the unit streams, the unit offsets,
    the sign+mantissa plane and 256 frequencies (2 bytes each)."""
    return enc.stream.size + 4 * enc.off16.size + enc.sign_mantissa.size + 512
