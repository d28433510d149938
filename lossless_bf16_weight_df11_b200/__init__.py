"""Python binding of the DF11 C ABI (``include/df11.h``, and the rANS
comparison variant of ``include/df11_rans.h``).

Argument marshalling only: every entry point of ``libdf11_b200.so`` is exposed
under its C name with the same arguments (device pointers and streams as
integers, host structs as ctypes structures).  All codec work happens in the
library's CUDA kernels and its C++ host code; there is no Python or CPU
fallback, and loading fails loudly if the library has not been built.

``lossless_bf16_weight_df11_b200.codec`` adds torch-tensor helpers that
allocate the buffers with PyTorch and call these entry points.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
# The product library; DF11_LIB may name another build of the same sources (the
# checked build, libdf11_b200_checked.so) to run the tests against it.
LIB_PATH = os.environ.get("DF11_LIB") or os.path.join(HERE, "libdf11_b200.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
HEADER = os.path.join(INCLUDE, "df11.h")
HEADERS = [HEADER, os.path.join(INCLUDE, "df11_rans.h")]

CHUNK_BITS = 64
BLOCK_CHUNKS = 256
GAP_BITS = 5
MAX_CODE_LEN = 32
MAX_N = 0xFFFFFFFF
MAX_BATCH = 32
TABLE_BITS = 11  # decode-table reach; the codec's default length cap
SEGMENT = 64     # DF11_SEGMENT: values per entry of the segment index

DF11_OK = 0
DF11_ERR_INVALID_ARG = 1
DF11_ERR_TOO_LARGE = 2
DF11_ERR_CUDA = 3
DF11_ERR_CORRUPT = 4
DF11_ERR_SYMBOL_NOT_IN_CODEBOOK = 5
DF11_ERR_TIMEOUT = 6
DF11_ERR_NO_DEVICE = 7
DF11_ERR_BOUNDS = 8


class df11_codebook(ctypes.Structure):
    _fields_ = [("len", ctypes.c_uint8 * 256), ("code", ctypes.c_uint32 * 256),
                ("max_len", ctypes.c_uint32), ("min_len", ctypes.c_uint32),
                ("n_symbols", ctypes.c_uint32), ("cap", ctypes.c_uint32)]


class df11_sizes(ctypes.Structure):
    _fields_ = [(name, ctypes.c_uint64) for name in (
        "n", "total_bits", "n_chunks", "n_blocks",
        "stream_bytes", "gaps_bytes", "block_pos_bytes", "sign_mantissa_bytes",
        "stored_bytes",
        "stream_alloc", "gaps_alloc", "block_pos_alloc", "sign_mantissa_alloc",
        "tables_bytes", "workspace_bytes", "run_index_bytes", "seg_index_bytes")]


class df11_matrix(ctypes.Structure):
    _fields_ = [("n", ctypes.c_uint64), ("total_bits", ctypes.c_uint64),
                ("stream", ctypes.c_void_p), ("gaps", ctypes.c_void_p),
                ("block_pos", ctypes.c_void_p), ("sign_mantissa", ctypes.c_void_p),
                ("tables", ctypes.c_void_p), ("min_len", ctypes.c_uint32),
                ("max_block_codes", ctypes.c_uint32), ("run_index", ctypes.c_void_p),
                ("seg_index", ctypes.c_void_p)]


class df11_encoded(ctypes.Structure):
    _fields_ = [("stream", ctypes.c_void_p), ("gaps", ctypes.c_void_p),
                ("block_pos", ctypes.c_void_p), ("sign_mantissa", ctypes.c_void_p),
                ("block_max", ctypes.c_void_p)]


class df11_matmul_io(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_uint32), ("cols", ctypes.c_uint32),
                ("x", ctypes.c_void_p), ("y", ctypes.c_void_p)]


class df11_host_matrix(ctypes.Structure):
    _fields_ = [("n", ctypes.c_uint64), ("total_bits", ctypes.c_uint64),
                ("cap", ctypes.c_uint32), ("max_block_codes", ctypes.c_uint32),
                ("ndim", ctypes.c_uint32), ("shape", ctypes.c_uint64 * 4),
                ("lengths", ctypes.c_void_p), ("gaps", ctypes.c_void_p),
                ("block_pos", ctypes.c_void_p), ("stream", ctypes.c_void_p),
                ("sign_mantissa", ctypes.c_void_p)]


FILE_VERSION = 1          # DF11_FILE_VERSION
FILE_HEADER_BYTES = 336   # DF11_FILE_HEADER_BYTES


class df11_rans_matrix(ctypes.Structure):
    _fields_ = [("n", ctypes.c_uint64), ("stream", ctypes.c_void_p), ("off16", ctypes.c_void_p),
                ("sign_mantissa", ctypes.c_void_p), ("tables", ctypes.c_void_p)]


class DF11Error(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {df11_status_string(status)} (status {status})")


_lock = threading.Lock()
_lib = None

_u64p = ctypes.POINTER(ctypes.c_uint64)
_vp = ctypes.c_void_p
_u64 = ctypes.c_uint64
_u32 = ctypes.c_uint32


def _declare(lib):
    sig = {
        "df11_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "df11_histogram": (ctypes.c_int, [_vp, _u64, _vp, _vp]),
        "df11_build_codebook": (ctypes.c_int, [_u64p, _u32, ctypes.POINTER(df11_codebook)]),
        "df11_encoded_sizes": (ctypes.c_int, [ctypes.POINTER(df11_codebook), _u64p, _u64,
                                              ctypes.POINTER(df11_sizes)]),
        "df11_tables_bytes": (ctypes.c_size_t, []),
        "df11_build_tables": (ctypes.c_int, [ctypes.POINTER(df11_codebook), _vp, ctypes.c_size_t]),
        "df11_encode": (ctypes.c_int, [_vp, _u64, ctypes.POINTER(df11_codebook), _u64,
                                       ctypes.POINTER(df11_encoded), _vp, ctypes.c_size_t, _vp, _vp]),
        "df11_decode": (ctypes.c_int, [ctypes.POINTER(df11_matrix), _vp, _vp, _vp]),
        "df11_decode_block_batch": (ctypes.c_int, [ctypes.POINTER(df11_matrix), _u32,
                                                   ctypes.POINTER(ctypes.c_void_p), _vp, _vp]),
        "df11_validate": (ctypes.c_int, [_u64, _u64, _u32, _vp, _u64, _vp, _u64]),
        "df11_encode_static_ws": (ctypes.c_int, [_vp, _u64, ctypes.POINTER(df11_codebook), _u64,
                                                 ctypes.POINTER(df11_encoded), _vp, _vp]),
        "df11_decode_matmul_batch": (ctypes.c_int, [ctypes.POINTER(df11_matrix),
                                                    ctypes.POINTER(df11_matmul_io), _u32, _u32,
                                                    _vp, _vp]),
        "df11_decode_gemm_batch": (ctypes.c_int, [ctypes.POINTER(df11_matrix),
                                                  ctypes.POINTER(df11_matmul_io), _u32, _u32,
                                                  _vp, _vp]),
        "df11_sizes_from_bits": (ctypes.c_int, [_u64, _u64, ctypes.POINTER(df11_sizes)]),
        "df11_file_bytes": (_u64, [_u64, _u64]),
        "df11_build_run_index": (ctypes.c_int, [ctypes.POINTER(df11_matrix), _vp, _vp, _vp]),
        "df11_build_segment_index": (ctypes.c_int, [ctypes.POINTER(df11_matrix), _vp, _vp, _vp]),
        "df11_write": (ctypes.c_int, [ctypes.POINTER(df11_host_matrix), _vp, _u64,
                                      ctypes.POINTER(ctypes.c_uint64)]),
        "df11_read": (ctypes.c_int, [_vp, _u64, ctypes.POINTER(df11_host_matrix)]),
        "df11_codebook_from_lengths": (ctypes.c_int, [_vp, _u32, ctypes.POINTER(df11_codebook)]),
        "df11_decode_host_scratch_bytes": (_u64, [ctypes.POINTER(df11_host_matrix), _u32]),
        "df11_decode_host_batch": (ctypes.c_int, [ctypes.POINTER(df11_host_matrix), _u32,
                                                  ctypes.POINTER(ctypes.c_void_p), _vp, _u64,
                                                  _vp, _vp]),
        "df11_build_codebook_device": (ctypes.c_int, [_vp, _u32, _vp, _vp, _vp, _vp, _vp]),
        "df11_encode_device_codebook": (ctypes.c_int, [_vp, _u64, _vp, _u64,
                                                       ctypes.POINTER(df11_encoded), _vp,
                                                       ctypes.c_size_t, _vp, _vp]),
        "df11_rans_freqs": (ctypes.c_int, [_u64p, ctypes.POINTER(ctypes.c_uint32)]),
        "df11_rans_build_tables": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _vp,
                                                  ctypes.c_size_t]),
        "df11_rans_units": (_u64, [_u64]),
        "df11_rans_validate": (ctypes.c_int, [_u64, _vp, _u64, _vp, _u64]),
        "df11_rans_encode_sizes": (ctypes.c_int, [_vp, _u64, _vp, _vp, _vp, _vp, _vp]),
        "df11_rans_encode": (ctypes.c_int, [_vp, _u64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "df11_rans_decode_batch": (ctypes.c_int, [ctypes.POINTER(df11_rans_matrix), _u32,
                                                  ctypes.POINTER(ctypes.c_void_p), _vp, _vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def library_path() -> str:
    return LIB_PATH


def load():
    """Load the built library; raise if it is missing (no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"DF11 CUDA library not built ({LIB_PATH}); run "
                    "`python -m lossless_bf16_weight_df11_b200.build` or __graft_entry__.build()")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def declared_functions() -> list[str]:
    """Names of the functions declared in the headers under include/."""
    names = set()
    for h in HEADERS:
        text = open(h).read()
        names |= set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(df11_\w+)\s*\(", text, re.M))
    return sorted(names)


# ------------------------------------------------------------- entry points


def df11_status_string(status: int) -> str:
    return load().df11_status_string(int(status)).decode()


def check(status: int, where: str = "df11") -> None:
    if status != DF11_OK:
        raise DF11Error(status, where)


def df11_histogram(d_w: int, n: int, d_hist256: int, stream: int = 0) -> int:
    return load().df11_histogram(d_w, n, d_hist256, stream)


def df11_build_codebook(hist256, cap: int = MAX_CODE_LEN):
    """hist256: 256 counts (any sequence).  Returns (status, df11_codebook)."""
    h = (ctypes.c_uint64 * 256)(*[int(x) for x in hist256])
    cb = df11_codebook()
    st = load().df11_build_codebook(h, cap, ctypes.byref(cb))
    return st, cb


def df11_encoded_sizes(cb: df11_codebook, hist256, n: int):
    h = (ctypes.c_uint64 * 256)(*[int(x) for x in hist256])
    out = df11_sizes()
    st = load().df11_encoded_sizes(ctypes.byref(cb), h, n, ctypes.byref(out))
    return st, out


def df11_tables_bytes() -> int:
    return int(load().df11_tables_bytes())


def df11_build_tables(cb: df11_codebook, h_tables: int, nbytes: int) -> int:
    return load().df11_build_tables(ctypes.byref(cb), h_tables, nbytes)


def df11_encode(d_w: int, n: int, cb: df11_codebook, total_bits: int, out: df11_encoded,
                d_workspace: int, workspace_bytes: int, d_status: int, stream: int = 0) -> int:
    return load().df11_encode(d_w, n, ctypes.byref(cb), total_bits, ctypes.byref(out),
                              d_workspace, workspace_bytes, d_status, stream)


def df11_decode(m: df11_matrix, d_out: int, d_status: int, stream: int = 0) -> int:
    return load().df11_decode(ctypes.byref(m), d_out, d_status, stream)


def df11_decode_block_batch(ms, d_outs, d_status: int, stream: int = 0) -> int:
    arr = (df11_matrix * len(ms))(*ms)
    outs = (ctypes.c_void_p * len(d_outs))(*[int(p) for p in d_outs])
    return load().df11_decode_block_batch(arr, len(ms), outs, d_status, stream)


MATMUL_MAX_BATCH = 8      # DF11_MATMUL_MAX_BATCH
MATMUL_MIN_COLS = 256     # DF11_MATMUL_MIN_COLS
GEMM_MAX_BATCH = 256      # DF11_GEMM_MAX_BATCH: activation rows per pass of the tensor-core path


def df11_decode_matmul_batch(ms, ios, batch: int, d_status: int, stream: int = 0) -> int:
    """y += x W^T for each (matrix, io) pair with W decoded on the fly; see
    include/df11.h."""
    arr = (df11_matrix * len(ms))(*ms)
    io = (df11_matmul_io * len(ios))(*ios)
    return load().df11_decode_matmul_batch(arr, io, len(ms), batch, d_status, stream)


def df11_decode_gemm_batch(ms, ios, batch: int, d_status: int, stream: int = 0) -> int:
    """y += x W^T on the tensor cores, W decoded through its segment index;
    see include/df11.h."""
    arr = (df11_matrix * len(ms))(*ms)
    io = (df11_matmul_io * len(ios))(*ios)
    return load().df11_decode_gemm_batch(arr, io, len(ms), batch, d_status, stream)


def df11_validate(n: int, total_bits: int, min_len: int, h_gaps: int, gaps_bytes: int,
                  h_block_pos: int, block_pos_count: int) -> int:
    return load().df11_validate(n, total_bits, min_len, h_gaps, gaps_bytes, h_block_pos,
                                block_pos_count)


def df11_sizes_from_bits(n: int, total_bits: int):
    out = df11_sizes()
    st = load().df11_sizes_from_bits(n, total_bits, ctypes.byref(out))
    return st, out


def df11_build_run_index(m: df11_matrix, d_run_index: int, d_status: int, stream: int = 0) -> int:
    """The matrix's run index (per pair of chunks, its first output within its
    block) into device memory; see include/df11.h."""
    return load().df11_build_run_index(ctypes.byref(m), d_run_index, d_status, stream)


def df11_build_segment_index(m: df11_matrix, d_seg_index: int, d_status: int,
                             stream: int = 0) -> int:
    """The matrix's segment index (the stream bit of every 64th code, then
    total_bits) into device memory; see include/df11.h."""
    return load().df11_build_segment_index(ctypes.byref(m), d_seg_index, d_status, stream)


def df11_file_bytes(n: int, total_bits: int) -> int:
    return int(load().df11_file_bytes(n, total_bits))


def df11_write(m: df11_host_matrix, buf: int, buf_bytes: int):
    """Serialise m into the host buffer at address buf; returns (status, bytes)."""
    written = ctypes.c_uint64(0)
    st = load().df11_write(ctypes.byref(m), buf, buf_bytes, ctypes.byref(written))
    return st, int(written.value)


def df11_read(buf: int, buf_bytes: int):
    """Parse a serialised matrix in the host buffer at address buf; returns
    (status, df11_host_matrix whose arrays point into that buffer)."""
    out = df11_host_matrix()
    st = load().df11_read(buf, buf_bytes, ctypes.byref(out))
    return st, out


def df11_decode_host_scratch_bytes(ms) -> int:
    """Device scratch df11_decode_host_batch needs for these host matrices
    (0 for an invalid one); see include/df11.h."""
    arr = (df11_host_matrix * len(ms))(*ms)
    return int(load().df11_decode_host_scratch_bytes(arr, len(ms)))


def df11_decode_host_batch(ms, h_outs, d_scratch: int, scratch_bytes: int, d_status: int,
                           stream: int = 0) -> int:
    """Decode host matrices into host buffers (addresses h_outs), copies and
    kernels pipelined over the device scratch; see include/df11.h."""
    arr = (df11_host_matrix * len(ms))(*ms)
    outs = (ctypes.c_void_p * len(h_outs))(*h_outs)
    return load().df11_decode_host_batch(arr, len(ms), outs, d_scratch, scratch_bytes, d_status,
                                         stream)


def df11_codebook_from_lengths(lengths: int, cap: int = MAX_CODE_LEN):
    """lengths: host address of 256 code lengths.  Returns (status, df11_codebook)."""
    cb = df11_codebook()
    st = load().df11_codebook_from_lengths(lengths, cap, ctypes.byref(cb))
    return st, cb


def df11_build_codebook_device(d_hist256: int, cap: int, d_cb: int, d_tables: int,
                               d_total_bits: int, d_status: int, stream: int = 0) -> int:
    """Codebook, decode tables and total_bits built on the device from a
    device histogram; see include/df11.h."""
    return load().df11_build_codebook_device(d_hist256, cap, d_cb, d_tables, d_total_bits,
                                             d_status, stream)


def df11_encode_device_codebook(d_w: int, n: int, d_cb: int, total_bits: int, out: df11_encoded,
                                d_workspace: int, workspace_bytes: int, d_status: int,
                                stream: int = 0) -> int:
    return load().df11_encode_device_codebook(d_w, n, d_cb, total_bits, ctypes.byref(out),
                                              d_workspace, workspace_bytes, d_status, stream)


CODEBOOK_BYTES = ctypes.sizeof(df11_codebook)   # 1296


STATIC_WS_MAX_N = 268431360  # DF11_STATIC_WS_MAX_N


def df11_encode_static_ws(d_w: int, n: int, cb: df11_codebook, total_bits: int, out: df11_encoded,
                          d_status: int, stream: int = 0) -> int:
    """df11_encode without a caller-provided workspace, for callers that cannot
    allocate device memory at the call site; see include/df11.h."""
    return load().df11_encode_static_ws(d_w, n, ctypes.byref(cb), total_bits, ctypes.byref(out),
                                        d_status, stream)


# ------------------------------------------------ rANS variant (df11_rans.h)

RANS_PROB_BITS = 12
RANS_UNIT = 16384
RANS_HEADER_BYTES = 144
RANS_TABLES_BYTES = 17408
RANS_MAX_BATCH = 32


def df11_rans_freqs(hist256):
    """Returns (status, list of 256 frequencies out of 4096)."""
    h = (ctypes.c_uint64 * 256)(*[int(x) for x in hist256])
    f = (ctypes.c_uint32 * 256)()
    st = load().df11_rans_freqs(h, f)
    return st, list(f)


def df11_rans_build_tables(freq, h_tables: int, nbytes: int) -> int:
    f = (ctypes.c_uint32 * 256)(*[int(x) for x in freq])
    return load().df11_rans_build_tables(f, h_tables, nbytes)


def df11_rans_units(n: int) -> int:
    return int(load().df11_rans_units(n))


def df11_rans_encode_sizes(d_w: int, n: int, d_tables: int, d_unit_words: int, d_off16: int,
                           d_status: int, stream: int = 0) -> int:
    return load().df11_rans_encode_sizes(d_w, n, d_tables, d_unit_words, d_off16, d_status, stream)


def df11_rans_encode(d_w: int, n: int, d_tables: int, d_unit_words: int, d_off16: int,
                     d_stream: int, d_sign_mantissa: int, d_status: int, stream: int = 0) -> int:
    return load().df11_rans_encode(d_w, n, d_tables, d_unit_words, d_off16, d_stream,
                                   d_sign_mantissa, d_status, stream)


def df11_rans_decode_batch(ms, d_outs, d_status: int, stream: int = 0) -> int:
    arr = (df11_rans_matrix * max(1, len(ms)))(*ms)
    outs = (ctypes.c_void_p * max(1, len(d_outs)))(*[int(p) for p in d_outs])
    return load().df11_rans_decode_batch(arr, len(ms), outs, d_status, stream)


def df11_rans_validate(n: int, h_stream: int, stream_bytes: int, h_off16: int,
                       off16_count: int) -> int:
    """Host check of rANS metadata (host copies); see include/df11_rans.h."""
    return load().df11_rans_validate(n, h_stream, stream_bytes, h_off16, off16_count)
