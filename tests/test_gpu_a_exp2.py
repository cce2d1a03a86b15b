"""The prefill kernel's FMA-pipe exponential (range reduction + cubic fit of 2^f on [0, 1))
against exact 2^x in FP64 and against CUDA's own exp2: bounded relative error over the whole
normal range, integer points, underflow and -inf inputs (the masked scores)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

REL_BOUND = 1.6e-4    # 7.5e-5 from the fit on [0, 1) plus FP32 rounding of the reduction


def _run(x):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    xt = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    y = fa4q.selftest_exp2(xt)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), xt


def test_exp2_relative_error_normal_range():
    import torch
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-126.0, 127.5, 1 << 20, dtype=np.float32),
                        rng.uniform(-20.0, 4.0, 1 << 20).astype(np.float32),
                        np.arange(-126, 128, dtype=np.float32),            # integers: f = 0
                        (np.arange(-126, 127, dtype=np.float32) + np.float32(0.99999994))])
    x = x[: len(x) // 2 * 2]
    y, xt = _run(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert np.all(np.isfinite(y))
    assert rel.max() <= REL_BOUND, f"max rel err {rel.max():.3e} at x={x[np.argmax(rel)]}"
    # against CUDA's exp2 (same bound: both sit within it of the exact value)
    yc = torch.exp2(xt).cpu().numpy().astype(np.float64)
    ok = yc > 0
    assert np.max(np.abs(y[ok] / yc[ok] - 1.0)) <= REL_BOUND + 1e-6


def test_exp2_underflow_and_masked_inputs():
    x = np.array([-127.0, -127.5, -130.0, -1e4, -np.inf, -np.inf, -3.0e38, -200.0], dtype=np.float32)
    y, _ = _run(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0.0)
    assert np.all(y < 2.0 ** -126), y          # E2M1 rounds all of these to 0
