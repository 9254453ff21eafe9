"""The softmax's FMA-pipe exp2 (Cody-Waite + degree-3 minimax, see
csrc/exp2_poly_fit.py) against float64 exp2 and against the hardware ex2.approx."""
import numpy as np
import pytest
import torch

import hybrid_sparse_linear_hf_b200 as hf

pytestmark = pytest.mark.gpu


def test_poly_exp2_error_bound():
    xs = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9, dtype=np.float64),
                         [0.0, -0.0, 1e-30, -1e-30, 7.999, -0.5, 0.5, -0.49999, 0.50001]]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    yp, ym = hf.hf_debug_exp2(x)
    torch.cuda.synchronize()
    ref = np.exp2(xs.astype(np.float64))
    rel_p = np.abs(yp.cpu().numpy().astype(np.float64) - ref) / ref
    rel_m = np.abs(ym.cpu().numpy().astype(np.float64) - ref) / ref
    assert rel_p.max() <= 1e-4, rel_p.max()      # 7.5e-5 fit + fp32 rounding
    assert rel_m.max() <= 1e-5, rel_m.max()      # hardware path, for scale
    assert np.all(yp.cpu().numpy() > 0)


def test_poly_exp2_underflow_and_masked():
    xs = np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    yp, ym = hf.hf_debug_exp2(torch.from_numpy(xs).cuda())
    torch.cuda.synchronize()
    assert np.all(yp.cpu().numpy() < 1e-37) and np.all(yp.cpu().numpy() >= 0)
    assert ym.cpu().numpy()[-1] == 0.0
