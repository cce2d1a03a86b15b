"""The bounded-wait error path: a wait that nothing satisfies expires, the kernel records a
timeout in the device status word and returns; the context stays usable."""
import pytest

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    assert fa4q.device_status()[0] == 0
    fa4q.selftest_wait_timeout(2000)
    code, detail = fa4q.device_status()
    assert code == 4 and detail & (1 << 4)
    assert fa4q.device_status() == (0, 0)
    x = torch.ones(4, device="cuda:0")
    assert float(x.sum()) == 4.0
