"""Query reordering along a Gilbert curve (paper §4.2; appendix "Spatial
reordering ablation"): the host order is pinned by what a space-filling
curve must satisfy, the device row gather against numpy indexing (gpu)."""
import numpy as np
import pytest

from adaptive_vector_quantized_avq_b200 import binding as bd
from adaptive_vector_quantized_avq_b200 import build as bl


@pytest.fixture(scope="module", autouse=True)
def _built():
    bl.build()


def _steps(order, cols):
    y, x = order // cols, order % cols
    return np.abs(np.diff(y)), np.abs(np.diff(x))


def test_gilbert_order_is_a_path_through_every_cell():
    for rows in range(1, 34):
        for cols in range(1, 34):
            o = bd.gilbert_order(rows, cols)
            assert np.array_equal(np.sort(o), np.arange(rows * cols)), (rows, cols)
            dy, dx = _steps(o, cols)
            assert not ((dy > 1) | (dx > 1)).any(), (rows, cols)      # no jumps
            diagonal = int(((dy == 1) & (dx == 1)).sum())
            assert diagonal <= 1, (rows, cols)                         # at most one diagonal step
            if rows % 2 == 0 and cols % 2 == 0:
                assert diagonal == 0, (rows, cols)                     # even grids: unit steps only


def test_gilbert_order_on_power_of_two_squares_is_a_hilbert_curve():
    """On 2^k x 2^k grids every aligned 2^j x 2^j block is visited
    contiguously (the defining recursion of the Hilbert curve)."""
    for k in (2, 3, 5):
        n = 1 << k
        o = bd.gilbert_order(n, n)
        y, x = o // n, o % n
        for j in range(1, k):
            b = 1 << j
            block = (y // b) * n + (x // b)
            runs = block.reshape(-1, b * b)
            assert np.all(runs == runs[:, :1]), (n, b)


def test_gilbert_tiles_are_compact():
    """Runs of T consecutive tokens cover compact regions: on a 64 x 64 grid
    with 128-token tiles the mean bounding-box diagonal is a fraction of the
    raster order's (whose tiles are 2 x 64 strips)."""
    rows = cols = 64
    T = 128
    def mean_extent(order):
        y, x = order // cols, order % cols
        ext = []
        for t in range(0, order.size, T):
            ys, xs = y[t:t + T], x[t:t + T]
            ext.append(np.hypot(ys.max() - ys.min() + 1, xs.max() - xs.min() + 1))
        return float(np.mean(ext))
    gil = mean_extent(bd.gilbert_order(rows, cols))
    raster = mean_extent(np.arange(rows * cols))
    assert gil < 0.4 * raster, (gil, raster)


def test_reorder_argument_errors():
    buf = np.empty(4, dtype=np.int32)
    assert bd.avq_gilbert_order(0, 4, buf) == -1
    assert bd.avq_gilbert_order(4, -1, buf) == -1
    assert bd.avq_gilbert_order(2, 2, 0) == -1
    A = 1 << 20
    s = bd.make_shape(1, 1, 16, 64, 1, 1, bd.AVQ_BF16)
    assert bd.avq_gather_rows(s, A + 8, A, A, stream=0) == -1      # misaligned source
    assert bd.avq_gather_rows(s, A, A, A + 2, stream=0) == -1      # misaligned perm
    assert bd.avq_gather_rows(bd.make_shape(1, 1, 16, 32, 1, 1, bd.AVQ_BF16), A, A, A, stream=0) == -1


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128)])
def test_gather_rows_gpu(dtype, d):
    import torch
    rng = np.random.default_rng(5)
    B, H, rows, cols = 2, 3, 13, 21
    N = rows * cols
    x = torch.from_numpy(rng.standard_normal((B, H, N, d)).astype(np.float32)).cuda()
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    order = bd.gilbert_order(rows, cols)
    perm = torch.from_numpy(order).cuda()
    y = bd.gather_rows(x, perm)
    torch.cuda.synchronize()
    assert torch.equal(y, x[:, :, perm.long()])                  # bit-exact gather
    inv = torch.empty_like(perm)
    inv[perm.long()] = torch.arange(N, dtype=torch.int32, device="cuda")
    assert torch.equal(bd.gather_rows(y, inv), x)                 # the inverse restores the order
    bad = perm.clone()
    bad[3] = N          # outside the sequence: the row is zeroed, nothing is read
    bad[5] = -1
    z = bd.gather_rows(x, bad)
    torch.cuda.synchronize()
    assert float(z[:, :, 3].abs().sum()) == 0.0 and float(z[:, :, 5].abs().sum()) == 0.0
    assert torch.equal(z[:, :, 4], x[:, :, perm[4].long()])
