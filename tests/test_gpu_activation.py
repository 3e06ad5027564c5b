"""The cell kernels' device tanh and sigmoid (exponential identities on the
special-function unit) against float64 and against CUDA's own tanhf/expf
(torch.tanh / torch.sigmoid): absolute error bound over the whole float range
the cells see, saturation and odd symmetry."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

BOUND = 6e-7   # absolute; well below the 1e-5 / 1e-6 residual tolerances of the workloads


def _eval(which, xs):
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    x = torch.from_numpy(xs).cuda()
    y = torch.empty_like(x)
    st = pn.pn_activation(which, x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == pn.PN_OK, pn.pn_last_error(None)
    return y.cpu().numpy(), x


def _grid():
    dense = np.linspace(-20.0, 20.0, 2_000_001, dtype=np.float64)
    tiny = np.concatenate([np.geomspace(1e-30, 1e-2, 20001), -np.geomspace(1e-30, 1e-2, 20001)])
    special = np.array([0.0, -0.0, 1e30, -1e30, 88.0, -88.0, 89.0, -104.0, 3.0e38, -3.0e38])
    return np.concatenate([dense, tiny, special]).astype(np.float32)


def test_tanh_error_bound():
    import torch
    xs = _grid()
    y, x = _eval(0, xs)
    ref = np.tanh(xs.astype(np.float64))
    assert np.isfinite(y).all()
    assert float(np.max(np.abs(y - ref))) <= BOUND
    cuda = torch.tanh(x).cpu().numpy().astype(np.float64)
    assert float(np.max(np.abs(y - cuda))) <= BOUND + 2e-7
    assert np.all(np.abs(y) <= 1.0)
    big = np.abs(xs) > 20
    np.testing.assert_array_equal(y[big], np.sign(xs[big]))


def test_sigmoid_error_bound():
    import torch
    xs = _grid()
    y, x = _eval(1, xs)
    ref = 1.0 / (1.0 + np.exp(-xs.astype(np.float64)))
    assert np.isfinite(y).all()
    assert float(np.max(np.abs(y - ref))) <= BOUND
    cuda = torch.sigmoid(x).cpu().numpy().astype(np.float64)
    assert float(np.max(np.abs(y - cuda))) <= BOUND + 2e-7
    assert np.all((y >= 0.0) & (y <= 1.0))
