"""fa4q_decode_noalloc: the decode entry point for callers that cannot allocate device
memory (a plug-in whose host framework owns all device memory, or a serving loop that must
not allocate).  Its split partials live in the library's static 8 MiB device array; this
checks it against fa4q_decode (caller workspace) on two calls in a row, within the decode
tests' tolerance, and that a request too large for the array is refused.

Collected last on purpose, so a run that stops at the first failure has run everything else.
"""
import numpy as np
import pytest

import synth
from fa4q_testlib import assert_close
from test_gpu_d_decode import build_cache

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L,splits", [(4160, 0), (2000, 3)])
def test_noalloc_decode_matches_workspace_decode_twice(L, splits):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    dw = synth.DecodeWorkload(95, f"noalloc_L{L}", B=2, Hq=8, Hkv=2, d=128, L=L)
    args, _, _, _ = build_cache(dw, dev)
    ref = fa4q.decode(*args, num_splits=splits).float().cpu().numpy()
    for _ in range(2):
        out = torch.full((dw.B, dw.Hq, dw.d), float("nan"), dtype=torch.bfloat16, device=dev)
        fa4q.decode_noalloc(*args, num_splits=splits, out=out)
        torch.cuda.synchronize()
        assert_close(out.float().cpu().numpy(), ref, mean_rel=5e-3, what="noalloc vs workspace decode")
    assert fa4q.device_status()[0] == 0


def test_noalloc_refuses_requests_beyond_the_static_array():
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    dw = synth.DecodeWorkload(96, "noalloc_big", B=2, Hq=8, Hkv=2, d=128, L=1000)
    args, _, _, _ = build_cache(dw, dev)
    # 2 * 8 * 130 * 4 = 8320 bytes per split: 2000 splits need 16.6 MB > 8 MiB
    with pytest.raises(fa4q.Fa4qError) as e:
        fa4q.decode_noalloc(*args, num_splits=2000)
    assert e.value.code == 2
