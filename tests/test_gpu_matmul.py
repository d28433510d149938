"""Fused decode -> matmul (df11_decode_matmul_batch): y = x W^T with W decoded
on the fly inside the decode kernel, never written as BF16.

Reference: W from the oracle (its decode of the oracle's own encoding for the
small cases; for the large ones the input itself, the oracle's round trip being
the identity, pinned in test_oracle_pins.py) and x, both BF16, widened to
float64, multiplied with numpy.

Tolerance, from the arithmetic: every product of two BF16 numbers is exact in
FP32 (8 + 8 significant bits <= 24), so the only error is the FP32 summation of
`cols` terms, whatever the order or tree of the additions:
|y - y_ref| <= (cols - 1) * 2^-24 * sum_c |W[r][c] x[c]| (to first order).  The
test allows (cols + 8) * 2^-24 * 1.01 times that sum.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def df11():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    import lossless_bf16_weight_df11_b200 as m
    return m


@pytest.fixture(scope="module")
def codec(df11):
    import lossless_bf16_weight_df11_b200.codec as c
    return c


def f64(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda()


def activations(batch: int, cols: int, seed: int) -> np.ndarray:
    g = np.random.default_rng(seed)
    return workloads.rne_to_bf16((g.standard_normal((batch, cols)) * 0.5).astype(np.float32))


def check_close(y: torch.Tensor, w_bits: np.ndarray, x_bits: np.ndarray):
    rows, cols = w_bits.shape
    W, X = f64(w_bits), f64(x_bits)
    ref = X @ W.T
    bound = (np.abs(X) @ np.abs(W).T) * (cols + 8) * U32 * 1.01
    got = y.double().cpu().numpy()
    err = np.abs(got - ref)
    worst = float((err - bound).max())
    assert worst <= 0.0, f"max excess over the summation bound: {worst:.3e}"


def run(codec, mats, xs_bits, batch):
    xs = [to_dev(x).view(torch.bfloat16).reshape(batch, -1) for x in xs_bits]
    return codec.matmul_block(mats, xs)


@pytest.mark.parametrize("batch", [1, 2, 3, 8])
@pytest.mark.parametrize("rows,cols,cap", [(64, 256, 11), (300, 1000, 11), (300, 1000, 12),
                                           (300, 1000, 32), (1, 4096, 11)])
def test_small_against_oracle_decode(codec, rows, cols, cap, batch):
    x = workloads.random_bf16(rows * cols, seed=rows * 7 + cols + cap).reshape(rows, cols)
    enc = oracle.encode(x.reshape(-1), cap=cap)
    w_ref = oracle.decode(enc, chunked=True).reshape(rows, cols)
    m = codec.compress(to_dev(x).reshape(rows, cols), cap=cap)
    xb = activations(batch, cols, seed=batch)
    (y,) = run(codec, [m], [xb], batch)
    torch.cuda.synchronize()
    check_close(y, w_ref, xb)


def test_codes_longer_than_the_table(codec):
    """Fibonacci exponent counts at cap 32: codes of up to 32 bits take the
    length search inside the fused kernel too."""
    x = workloads.fibonacci_exponents(30)[: 2048 * 512].reshape(2048, 512)
    m = codec.compress(to_dev(x).reshape(2048, 512), cap=32)
    assert int(m.codebook.max_len) > 11
    xb = activations(4, 512, seed=4)
    (y,) = run(codec, [m], [xb], 4)
    check_close(y, x, xb)


@pytest.mark.parametrize("batch", [1, 8])
def test_matrix_4096x4096(codec, batch):
    x = workloads.matrix(2, 0)
    m = codec.compress(to_dev(x).reshape(4096, 4096))
    xb = activations(batch, 4096, seed=10 + batch)
    (y,) = run(codec, [m], [xb], batch)
    check_close(y, x, xb)


def test_llama3_8b_block_batched(codec):
    """The seven matrices of the Llama-3-8B-shaped block in one launch (per-matrix
    codebooks), batch 4."""
    names = workloads.WORKLOADS[3][1]
    mats, ws, xs = [], [], []
    for i, (_, shape) in enumerate(names):
        w = workloads.matrix(3, i).reshape(shape)
        mats.append(codec.compress(to_dev(w).reshape(shape)))
        ws.append(w)
        xs.append(activations(4, shape[1], seed=100 + i))
    ys = run(codec, mats, xs, 4)
    for y, w, xb in zip(ys, ws, xs):
        check_close(y, w, xb)


def test_accumulates_into_y(codec):
    x = workloads.random_bf16(256 * 512, seed=5).reshape(256, 512)
    m = codec.compress(to_dev(x).reshape(256, 512))
    xb = activations(2, 512, seed=6)
    xt = to_dev(xb).view(torch.bfloat16).reshape(2, 512)
    y = torch.full((2, 256), 1.5, dtype=torch.float32, device="cuda")
    codec.matmul_block([m], [xt], [y])
    y -= 1.5
    check_close(y, x, xb)


def test_corrupt_positions_reported(codec):
    x = workloads.random_bf16(512 * 4096, seed=9).reshape(512, 4096)
    m = codec.compress(to_dev(x).reshape(512, 4096))
    m.block_pos[3] += 5
    xt = to_dev(activations(1, 4096, seed=1)).view(torch.bfloat16).reshape(1, 4096)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codec.matmul_block([m], [xt], status=status)
    assert int(status.item()) == 4  # DF11_ERR_CORRUPT


def test_rejects_bad_shapes(df11, codec):
    x = workloads.random_bf16(256 * 1024, seed=2)
    m = codec.compress(to_dev(x).reshape(256, 1024))
    y = torch.zeros(8, 4096, dtype=torch.float32, device="cuda")
    xb = torch.zeros(8, 4096, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream

    def call(rows, cols, batch):
        io = df11.df11_matmul_io(rows=rows, cols=cols, x=xb.data_ptr(), y=y.data_ptr())
        return df11.df11_decode_matmul_batch([m.abi()], [io], batch, status.data_ptr(), stream)

    assert call(256, 1024, 1) == df11.DF11_OK
    torch.cuda.synchronize()
    assert call(128, 1024, 1) == df11.DF11_ERR_INVALID_ARG    # rows * cols != n
    assert call(2048, 128, 1) == df11.DF11_ERR_INVALID_ARG    # cols below 256
    assert call(256, 1024, 0) == df11.DF11_ERR_INVALID_ARG
    assert call(256, 1024, 9) == df11.DF11_ERR_INVALID_ARG
    # cols not a multiple of 8 (a 258 x 1002 matrix)
    x2 = workloads.random_bf16(258 * 1002, seed=3)
    m2 = codec.compress(to_dev(x2).reshape(258, 1002))
    io = df11.df11_matmul_io(rows=258, cols=1002, x=xb.data_ptr(), y=y.data_ptr())
    assert df11.df11_decode_matmul_batch([m2.abi()], [io], 1, status.data_ptr(),
                                         stream) == df11.DF11_ERR_INVALID_ARG


def test_more_matrices_than_one_launch(codec):
    """40 matrices (DF11_MAX_BATCH = 32 per launch), batch 2."""
    shapes = [(16 + 8 * i, 256 + 64 * (i % 5)) for i in range(40)]
    xs = [workloads.random_bf16(r * c, seed=900 + i).reshape(r, c) for i, (r, c) in enumerate(shapes)]
    mats = codec.compress_block([to_dev(x).reshape(x.shape) for x in xs])
    acts = [activations(2, c, seed=40 + i) for i, (_, c) in enumerate(shapes)]
    ys = run(codec, mats, acts, 2)
    for y, w, xb in zip(ys, xs, acts):
        check_close(y, w, xb)
