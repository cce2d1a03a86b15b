"""One BF16 tensor-core MMA (kind::f16) through the operand layouts of the full-precision
tiles of the hybrid prefill, against an FP64 product: pins the instruction descriptor, the
128-byte swizzle and the K-major / MN-major shared-memory descriptors."""
import numpy as np
import pytest

from fa4q_testlib import to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K,b_mn", [(64, 128, 0), (128, 128, 0), (16, 64, 0), (64, 64, 0),
                                      (128, 64, 1), (64, 64, 1), (128, 128, 1)])
def test_bf16_mma(N, K, b_mn):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    import synth
    rng = np.random.default_rng(N * 100 + K + b_mn)
    a = synth.round_to_bf16(rng.normal(size=(128, K)).astype(np.float32))
    b = synth.round_to_bf16(rng.normal(size=(K, N) if b_mn else (N, K)).astype(np.float32))
    dev = torch.device("cuda:0")
    got = fa4q.selftest_bf16_mma(to_dev_bf16(a, dev), to_dev_bf16(b, dev), N, K, b_mn).cpu().numpy()
    ref = a.astype(np.float64) @ (b.astype(np.float64) if b_mn else b.astype(np.float64).T)
    bound = 1e-5 * (np.abs(a).astype(np.float64) @ (np.abs(b) if b_mn else np.abs(b).T)) + 1e-6
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"{(err > bound).sum()} wrong, max err {err.max():.3g}"
    assert fa4q.device_status()[0] == 0
