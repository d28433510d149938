"""Fused decode -> tensor-core GEMM (df11_decode_gemm_batch): y += x W^T with W
decoded through its segment index straight into the operand tiles of
tcgen05.mma, never written as BF16.

Reference: W from the oracle (its decode of the oracle's own encoding for the
small cases; for the large ones the input itself, the oracle's round trip being
the identity, pinned in test_oracle_pins.py) and x, both BF16, widened to
float64, multiplied with numpy.

Tolerance, from the arithmetic: every product of two BF16 numbers is exact in
FP32, so the error is the FP32 accumulation of `cols` terms.  The tensor cores'
accumulation order and rounding of the intermediate sums are not specified, so
the bound allows one unit in the last place (2^-23 relative) per addition
rather than half of one: |y - y_ref| <= (cols + 8) * 2^-23 * sum_c |W[r][c]
x[c]|, times 1.01.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

ULP = 2.0 ** -23
CORRUPT, INVALID = 4, 1


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


def check_close(got: np.ndarray, w_bits: np.ndarray, x_bits: np.ndarray, y0=None):
    cols = w_bits.shape[1]
    W, X = f64(w_bits), f64(x_bits)
    ref = X @ W.T + (0.0 if y0 is None else y0)
    bound = (np.abs(X) @ np.abs(W).T) * (cols + 8) * ULP * 1.01
    if y0 is not None:
        bound += np.abs(y0) * ULP
    err = np.abs(got - ref)
    worst = float((err - bound).max())
    assert worst <= 0.0, f"max excess over the summation bound: {worst:.3e}"


def gemm(codec, mats, xs_bits, batch, ys=None):
    xs = [to_dev(x).view(torch.bfloat16).reshape(batch, -1) for x in xs_bits]
    return codec.gemm_block(mats, xs, ys)


@pytest.mark.parametrize("batch", [1, 16, 128, 129, 256, 300])
@pytest.mark.parametrize("rows,cols,cap", [(128, 64, 11), (300, 256, 11), (300, 256, 32),
                                           (64, 1024, 12), (1, 4096, 11)])
def test_small_against_oracle_decode(codec, rows, cols, cap, batch):
    """One and several M tiles (129 and 256 rows: two; 300: two passes), a
    ragged N tile (300 and 64 rows of W), one k step (64 columns), codes past
    the decode table (cap 12 and 32)."""
    x = workloads.random_bf16(rows * cols, seed=rows * 5 + cols + cap).reshape(rows, cols)
    enc = oracle.encode(x.reshape(-1), cap=cap)
    w_ref = oracle.decode(enc, chunked=True).reshape(rows, cols)
    m = codec.compress(to_dev(x).reshape(rows, cols), cap=cap)
    xb = activations(batch, cols, seed=batch + cols)
    (y,) = gemm(codec, [m], [xb], batch)
    check_close(y.double().cpu().numpy(), w_ref, xb)


def test_accumulates_into_y(codec):
    rows, cols, batch = 200, 512, 40
    x = workloads.random_bf16(rows * cols, seed=91).reshape(rows, cols)
    m = codec.compress(to_dev(x).reshape(rows, cols))
    xb = activations(batch, cols, seed=92)
    y0 = np.random.default_rng(93).standard_normal((batch, rows)).astype(np.float32)
    (y,) = gemm(codec, [m], [xb], batch, [torch.from_numpy(y0).cuda()])
    check_close(y.double().cpu().numpy(), x, xb, y0.astype(np.float64))


@pytest.mark.parametrize("batch", [64, 256])
def test_block_of_seven_matrices(codec, batch):
    """The Llama-3-8B-shaped block in one call (seven matrices, per-matrix
    codebooks), checked on 48 sampled rows of W per matrix."""
    wid = 3
    names = workloads.WORKLOADS[wid][1]
    xs_w = [workloads.matrix(wid, i) for i in range(len(names))]
    mats = [codec.compress(to_dev(w).reshape(w.shape)) for w in xs_w]
    xb = [activations(batch, w.shape[1], seed=7 + i) for i, w in enumerate(xs_w)]
    ys = gemm(codec, mats, xb, batch)
    g = np.random.default_rng(5)
    for w, x, y in zip(xs_w, xb, ys):
        r = np.sort(g.choice(w.shape[0], 48, replace=False))
        check_close(y.double().cpu().numpy()[:, r], w[r], x)


def test_corrupt_segment_index_is_reported_without_fault(codec):
    rows, cols, batch = 256, 1024, 32
    x = workloads.random_bf16(rows * cols, seed=61).reshape(rows, cols)
    m = codec.compress(to_dev(x).reshape(rows, cols))
    xb = activations(batch, cols, seed=62)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    si = m.seg_index.clone()
    for k, v in ((3, 1), (100, -2), (rows * cols // 64, 5), (17, 1 << 30)):
        m.seg_index[k] = max(0, min(int(si[k]) + v, (1 << 31) - 1))
        status.zero_()
        codec.gemm_block([m], [to_dev(xb).view(torch.bfloat16).reshape(batch, cols)], status=status)
        assert int(status.item()) == CORRUPT, (k, v)
        m.seg_index.copy_(si)
    status.zero_()
    (y,) = codec.gemm_block([m], [to_dev(xb).view(torch.bfloat16).reshape(batch, cols)],
                            status=status)
    assert int(status.item()) == 0
    check_close(y.double().cpu().numpy(), x, xb)


def test_rejects_invalid_arguments(df11, codec):
    rows, cols = 64, 96  # cols not a multiple of 64
    x = workloads.random_bf16(rows * cols, seed=71).reshape(rows, cols)
    m = codec.compress(to_dev(x).reshape(rows, cols))
    xd = to_dev(activations(4, cols, 72)).view(torch.bfloat16).reshape(4, cols)
    y = torch.zeros(4, rows, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    io = df11.df11_matmul_io(rows=rows, cols=cols, x=xd.data_ptr(), y=y.data_ptr())
    assert df11.df11_decode_gemm_batch([m.abi()], [io], 4, status.data_ptr(), 0) == INVALID
    x2 = workloads.random_bf16(64 * 128, seed=73).reshape(64, 128)
    m2 = codec.compress(to_dev(x2).reshape(64, 128))
    xd2 = to_dev(activations(4, 128, 74)).view(torch.bfloat16).reshape(4, 128)
    io2 = df11.df11_matmul_io(rows=64, cols=128, x=xd2.data_ptr(), y=y.data_ptr())
    assert df11.df11_decode_gemm_batch([m2.abi(True, False)], [io2], 4, status.data_ptr(), 0) == INVALID
    assert df11.df11_decode_gemm_batch([m2.abi()], [io2], 0, status.data_ptr(), 0) == INVALID
    assert int(status.item()) == 0
