"""fa4q_decode_noalloc: the decode entry point for callers that cannot allocate device
memory (a plug-in whose host framework owns all device memory, or a serving loop that must
not allocate).  Its split partials live in the library's static 8 MiB device array.

It runs the same kernels as fa4q_decode with the same split count, so its output must be
bit-identical to fa4q_decode's with a caller workspace.  Each check follows a call on other
data, so partials left in the shared array by an earlier call would show.

Collected last on purpose, so a run that stops at the first failure has run everything else.
"""
import numpy as np
import pytest

import synth
from test_gpu_d_decode import build_cache

pytestmark = pytest.mark.gpu


def _noalloc(args, dw, splits):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    out = torch.full((dw.B, dw.Hq, dw.d), float("nan"), dtype=torch.bfloat16, device=args[0].device)
    fa4q.decode_noalloc(*args, num_splits=splits, out=out)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("L,splits", [(4160, 0), (2000, 3)])
def test_noalloc_decode_matches_workspace_decode_twice(L, splits):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    dw = synth.DecodeWorkload(95, f"noalloc_L{L}", B=2, Hq=8, Hkv=2, d=128, L=L)
    other = synth.DecodeWorkload(99, "noalloc_other", B=3, Hq=8, Hkv=2, d=128, L=1500)
    args, _, _, _ = build_cache(dw, dev)
    args_other, _, _, _ = build_cache(other, dev)
    ref = fa4q.decode(*args, num_splits=splits).float().cpu().numpy()
    for _ in range(2):
        _noalloc(args_other, other, 0)          # leaves other partials in the static array
        got = _noalloc(args, dw, splits)
        assert np.array_equal(got, ref), np.nanmax(np.abs(got - ref))
    assert fa4q.device_status()[0] == 0


def test_noalloc_lowers_the_automatic_split_count_to_fit_the_array():
    """128 sequences x 64 query heads: the automatic split count (2) needs 8.5 MB of partials,
    so the call runs 1 split; its output equals fa4q_decode's with num_splits = 1."""
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    dev = torch.device("cuda:0")
    dw = synth.DecodeWorkload(90, "noalloc_lowered", B=128, Hq=64, Hkv=8, d=128, L=400)
    per_split = dw.B * dw.Hq * (dw.d + 2) * 4
    assert 1 * per_split <= (8 << 20) < 2 * per_split
    args, _, _, _ = build_cache(dw, dev)
    ref = fa4q.decode(*args, num_splits=1).float().cpu().numpy()
    for _ in range(2):
        got = _noalloc(args, dw, 0)
        assert np.array_equal(got, ref), np.nanmax(np.abs(got - ref))
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
