"""Seeded synthetic BF16 weight matrices for the DF11 workloads.

This module only draws random numbers and rounds them to BF16; it holds none of
the codec's arithmetic.  Both the CPU oracle (through the tests) and the CUDA
library (through the tests and ``bench.py``) take their inputs from here.

The page being implemented ("DFloat11: Nén suy luận GPU không mất dữ liệu, giảm
LLM xuống còn 70% kích thước", vi.news.hada.io/topic?id=20542, section "Kết quả
đánh giá và hiệu quả thực tế") measures trained checkpoints (Llama 3, Qwen 3,
Mistral 3, ...).  None are available here, so each workload is a synthetic
stand-in with the shapes of the models named and a weight distribution of the
same kind (zero-mean, small scale, heavy or light tails).

Recipe (every value is reproducible from its key):
  * a matrix is cut into pieces of ``PIECE`` elements; piece ``p`` of matrix
    ``i`` of workload seed ``s`` is drawn by
    ``numpy.random.Generator(PCG64(SeedSequence([s, i, p])))``;
    pieces are filled in parallel threads, so the result does not depend on the
    thread count;
  * fp32 samples are rounded to BF16 with round-to-nearest-even (no NaN is ever
    produced, so the rounding needs no NaN case).

Workloads (sizes are element counts; matrices are out_features x in_features):
  1  "matrix_256x1024"    one 256x1024 matrix, N(0, 0.02), seed 0
  2  "matrix_4096x4096"   one 4096x4096 matrix, N(0, 0.02); exactly
                          round(0.001 n) distinct entries chosen uniformly and
                          multiplied by 20 before rounding, seed 1
  3  "llama3_8b_block"    q,o 4096x4096; k,v 1024x4096; gate,up 14336x4096;
                          down 4096x14336; N(0, 1/sqrt(in_features)), seed 3
  4  "stress_64Mi"        67,108,864 values: 98% magnitude 2^U(-40,4),
                          1% signed zeros, 1% subnormals (exponent 0, mantissa
                          uniform in 1..127), random signs, seed 4
  5  "llama3_70b_block"   q,o 8192x8192; k,v 1024x8192; gate,up 28672x8192;
                          down 8192x28672; Student-t(nu=4) x 0.015, seed 5
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

PIECE = 1 << 22

MATRIX_NAMES = ("q", "o", "k", "v", "gate", "up", "down")

WORKLOADS = {
    1: ("matrix_256x1024", [("w", (256, 1024))]),
    2: ("matrix_4096x4096", [("w", (4096, 4096))]),
    3: ("llama3_8b_block", [("q", (4096, 4096)), ("o", (4096, 4096)), ("k", (1024, 4096)),
                            ("v", (1024, 4096)), ("gate", (14336, 4096)), ("up", (14336, 4096)),
                            ("down", (4096, 14336))]),
    4: ("stress_64Mi", [("w", (1 << 26,))]),
    5: ("llama3_70b_block", [("q", (8192, 8192)), ("o", (8192, 8192)), ("k", (1024, 8192)),
                             ("v", (1024, 8192)), ("gate", (28672, 8192)), ("up", (28672, 8192)),
                             ("down", (8192, 28672))]),
}
SEEDS = {1: 0, 2: 1, 3: 3, 4: 4, 5: 5}


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def rne_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> BF16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    out = np.empty(u.shape, np.uint16)
    step = 1 << 22
    flat_u, flat_o = u.reshape(-1), out.reshape(-1)
    for a in range(0, flat_u.size, step):
        v = flat_u[a:a + step].astype(np.uint64)
        flat_o[a:a + step] = ((v + 0x7FFF + ((v >> 16) & 1)) >> 16).astype(np.uint16)
    return out


def _fill(n: int, key, draw) -> np.ndarray:
    """Fill n BF16 values piece by piece; draw(gen, size) -> fp32 samples."""
    out = np.empty(n, np.uint16)
    pieces = (n + PIECE - 1) // PIECE

    def one(p):
        a, b = p * PIECE, min(n, (p + 1) * PIECE)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key) + [p])))
        out[a:b] = rne_to_bf16(draw(g, b - a))

    if pieces <= 1:
        for p in range(pieces):
            one(p)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(pieces)))
    return out


def _normal(std):
    return lambda g, k: (g.standard_normal(k, dtype=np.float32) * np.float32(std))


def _student_t(nu, scale):
    return lambda g, k: (g.standard_t(nu, k) * scale).astype(np.float32)


def _stress_draw(g, k):
    """98% log-uniform magnitudes over 2^-40..2^4, 1% signed zeros, 1% subnormals."""
    cat = g.random(k)
    sign = g.integers(0, 2, k, dtype=np.uint32) << 31
    mag = np.exp2(g.uniform(-40.0, 4.0, k)).astype(np.float32).view(np.uint32)
    # BF16 subnormal: exponent 0, mantissa m in 1..127 -> fp32 bits m << 16 round exactly
    sub = g.integers(1, 128, k, dtype=np.uint32) << 16
    bits = np.where(cat < 0.98, mag, np.where(cat < 0.99, np.uint32(0), sub)) | sign
    return bits.astype(np.uint32).view(np.float32)


def matrix(workload: int, index: int) -> np.ndarray:
    """BF16 bit patterns (uint16) of matrix ``index`` of ``workload``."""
    name, mats = WORKLOADS[workload]
    mname, shape = mats[index]
    n = int(np.prod(shape))
    seed = SEEDS[workload]
    key = (seed, index)
    if workload in (1, 2):
        w = _fill(n, key, _normal(0.02))
        if workload == 2:
            k = int(round(0.001 * n))
            g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, index, 1 << 30])))
            idx = g.choice(n, size=k, replace=False)
            # redraw those entries' fp32 values with the same piece generators would be
            # awkward; instead scale the rounded value's fp32 original: regenerate exactly
            x = _regen_fp32(n, key, _normal(0.02), idx)
            w[idx] = rne_to_bf16(x * np.float32(20.0))
        return w.reshape(shape)
    if workload == 3:
        fan_in = shape[-1]
        return _fill(n, key, _normal(1.0 / np.sqrt(fan_in))).reshape(shape)
    if workload == 4:
        return _fill(n, key, _stress_draw).reshape(shape)
    if workload == 5:
        return _fill(n, key, _student_t(4.0, 0.015)).reshape(shape)
    raise KeyError(workload)


def _regen_fp32(n: int, key, draw, idx: np.ndarray) -> np.ndarray:
    """The fp32 samples (before rounding) at positions idx, redrawn piece by piece."""
    out = np.empty(idx.size, np.float32)
    order = np.argsort(idx, kind="stable")
    sidx = idx[order]
    pieces = (n + PIECE - 1) // PIECE
    for p in range(pieces):
        a, b = p * PIECE, min(n, (p + 1) * PIECE)
        lo, hi = np.searchsorted(sidx, a), np.searchsorted(sidx, b)
        if lo == hi:
            continue
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key) + [p])))
        x = draw(g, b - a)
        out[order[lo:hi]] = x[sidx[lo:hi] - a]
    return out


def workload(workload_id: int):
    """[(name, uint16 matrix)] for every matrix of the workload."""
    return [(m[0], matrix(workload_id, i)) for i, m in enumerate(WORKLOADS[workload_id][1])]


def workload_name(workload_id: int) -> str:
    return WORKLOADS[workload_id][0]


def workload_sizes(workload_id: int):
    return [int(np.prod(s)) for _, s in WORKLOADS[workload_id][1]]


# ------------------------------------------------------------ edge-case inputs


def all_patterns() -> np.ndarray:
    """Every one of the 65,536 BF16 bit patterns, in order."""
    return np.arange(65536, dtype=np.uint32).astype(np.uint16)


def shuffled_patterns(copies: int = 4, seed: int = 7) -> np.ndarray:
    g = np.random.default_rng(seed)
    x = np.tile(all_patterns(), copies)
    g.shuffle(x)
    return x


def fibonacci_counts(k: int) -> list[int]:
    """F_1..F_k = 1, 1, 2, 3, 5, ..."""
    f = [1, 1]
    while len(f) < k:
        f.append(f[-1] + f[-2])
    return f[:k]


def fibonacci_exponents(k: int = 34, seed: int = 11, first_exponent: int = 100) -> np.ndarray:
    """BF16 words whose exponent counts are F_1..F_k (exponent first_exponent+i
    occurs F_{i+1} times), shuffled, with random sign and mantissa.  With k=34
    there are 14,930,351 values and an unconstrained Huffman code is 33 bits
    long, one more than the cap of 32."""
    g = np.random.default_rng(seed)
    counts = fibonacci_counts(k)
    e = np.repeat(np.arange(first_exponent, first_exponent + k, dtype=np.uint16),
                  np.asarray(counts, dtype=np.int64))
    g.shuffle(e)
    sm = g.integers(0, 256, e.size, dtype=np.uint16)
    return (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)


def random_bf16(n: int, seed: int, std: float = 0.02) -> np.ndarray:
    g = np.random.default_rng(seed)
    return rne_to_bf16(g.standard_normal(n, dtype=np.float32) * np.float32(std))


def constant(n: int, value: int = 0x3C00) -> np.ndarray:
    return np.full(n, value, dtype=np.uint16)
