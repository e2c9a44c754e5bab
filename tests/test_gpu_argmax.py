"""bi_argmax on the GPU: the greedy token is the largest logit, lowest index
on exact ties, NaN above every number (first NaN wins), whatever the row's
batch position or the other rows -- the near-tie flips the Metal-vs-CUDA
post reports are exactly where an order-dependent tie-break would show.
Checked against the oracle's argmax (numpy: first maximum, NaN first)."""
import numpy as np
import pytest
import torch

from oracle import fp64
from tests.gpu_common import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bi(cuda_device):
    from invariant_deterministic_03_b200 import bi as mod
    return mod


def _argmax(bi, x):
    idx = torch.empty(x.shape[0], dtype=torch.int32, device="cuda:0")
    bi.bi_argmax(x, idx)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


def _rows(V):
    """Rows whose maximum repeats at indices that fall in the same thread,
    in different threads of one warp, in different warps and in different
    strides of the 256-thread loop; plus NaN, +inf and all -inf rows."""
    rng = np.random.default_rng(V)
    rows = []
    for ties in ([3, 7], [0, V - 1], [5, 5 + 256], [31, 32], [255, 256, 511], [V // 2, V // 3, V - 2],
                 [1, 33, 65, 97, 129]):
        r = rng.standard_normal(V).astype(np.float32)
        for t in ties:
            r[t % V] = 9.5
        rows.append(r)
    r = rng.standard_normal(V).astype(np.float32)
    r[[V - 1, min(4, V - 2), V // 2]] = np.nan
    rows.append(r)                                   # the first NaN wins
    r = rng.standard_normal(V).astype(np.float32)
    r[min(7, V - 1)] = np.inf
    r[V - 3] = np.nan
    rows.append(r)                                   # NaN above +inf
    rows.append(np.full(V, -np.inf, np.float32))     # all -inf: index 0
    r = np.zeros(V, np.float32)
    r[V - 1] = np.float32(1.0) + np.float32(2.0 ** -23)
    r[2] = 1.0
    rows.append(r)                                   # one ulp apart: the larger wins
    rows.append(rng.standard_normal(V).astype(np.float32))
    return np.stack(rows)


@pytest.mark.parametrize("V", [32000, 257, 7])
def test_argmax_ties_nan_and_oracle(bi, V):
    x = _rows(V)
    got = _argmax(bi, dev(torch.from_numpy(x)))
    np.testing.assert_array_equal(got, fp64.argmax_first(x))


def test_argmax_row_alone_and_permuted(bi):
    x = _rows(32000)
    full = _argmax(bi, dev(torch.from_numpy(x)))
    for i in range(x.shape[0]):
        assert _argmax(bi, dev(torch.from_numpy(x[i:i + 1])))[0] == full[i]
    perm = np.random.default_rng(0).permutation(x.shape[0])
    np.testing.assert_array_equal(_argmax(bi, dev(torch.from_numpy(x[perm]))), full[perm])
