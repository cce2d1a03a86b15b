"""Host-side checks of the C ABI library: it loads without a GPU, exports every symbol the
header declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__.build()
    import microscaled_fp4_flashattention_b200 as fa4q
    return fa4q.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "fa4q.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa4q_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    import microscaled_fp4_flashattention_b200 as fa4q
    assert sorted(fa4q.EXPORTED) == names


def test_status_strings_and_version(L):
    assert L.fa4q_status_string(0) == b"ok"
    assert L.fa4q_status_string(4).startswith(b"a bounded")
    assert L.fa4q_version() == 100


def test_sf_tiled_bytes(L):
    assert L.fa4q_sf_tiled_bytes(128, 128, 0) == 2 * 512
    assert L.fa4q_sf_tiled_bytes(128, 128, 1) == 512
    assert L.fa4q_sf_tiled_bytes(129, 64, 0) == 2 * 2 * 512
    assert L.fa4q_sf_tiled_bytes(4096, 128, 0) == 32 * 2 * 512
    assert L.fa4q_sf_tiled_bytes(0, 128, 0) == 0


def test_argument_errors_without_gpu(L):
    P = ctypes.c_void_p
    fake = P(0x1000)  # never dereferenced: validation fails first
    # null input
    assert L.fa4q_quantize(None, 1, 16, 16, 16, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    # bad format / axis / misaligned stride
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 7, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 0, 5, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    assert L.fa4q_quantize(fake, 1, 16, 16, 12, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    # cols not a multiple of the block
    assert L.fa4q_quantize(fake, 1, 16, 24, 24, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 2
    # negative qmax, non-positive tensor scale
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 0, 0, -1.0, 1.0, None, 1, 1, 1, fake, fake, None) == 1
    assert L.fa4q_quantize(fake, 1, 16, 16, 16, 0, 0, 0.0, 0.0, None, 1, 1, 1, fake, fake, None) == 1
    # empty input is a no-op
    assert L.fa4q_quantize(fake, 0, 16, 16, 16, 0, 0, 0.0, 1.0, None, 1, 1, 1, fake, fake, None) == 0
    F = ctypes.c_float
    # attention: unsupported head dim, GQA mismatch, causal with S_q != S_k
    args = [fake] * 6 + [F(1), F(1), F(1)]
    assert L.fa4q_attn_fwd(*args, 1, 4, 4, 128, 128, 96, 0, F(0), 0, F(0), fake, 1, None, None) == 2
    assert L.fa4q_attn_fwd(*args, 1, 6, 4, 128, 128, 128, 0, F(0), 0, F(0), fake, 1, None, None) == 1
    assert L.fa4q_attn_fwd(*args, 1, 4, 4, 128, 256, 128, 0, F(0), 1, F(0), fake, 1, None, None) == 1
    # conditional rescaling: threshold out of range; NVFP4 P with a kept reference
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 1, F(0), 0, F(0), 31, 0, fake, 1, None, None) == 1
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 1, F(0), 0, F(0), -1, 0, fake, 1, None, None) == 1
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 0, F(0), 0, F(0), 8, 0, fake, 1, None, None) == 2
    # inconsistent-normaliser flag must be 0 or 1
    assert L.fa4q_attn_fwd_ex(*args, 1, 4, 4, 128, 128, 128, 1, F(0), 0, F(0), 0, 2, fake, 1, None, None) == 1
    # rotated quantisation: head dims other than 64 / 128
    assert L.fa4q_quantize_rotated(fake, 1, 16, 96, 96, 0, F(0), F(1), None, 1, 1, 1, fake, fake, None) == 2
    assert L.fa4q_quantize_rotated(None, 1, 16, 128, 128, 0, F(0), F(1), None, 1, 1, 1, fake, fake, None) == 1
    # decode: group too large, workspace too small
    dargs = [fake] * 14
    assert L.fa4q_decode(*dargs, 1, 32, 2, 128, 4, 0, 0, 0, F(1), F(1), F(0), fake, fake, 1 << 30, 0, None) == 2
    assert L.fa4q_decode(*dargs, 1, 8, 2, 128, 4, 0, 0, 0, F(1), F(1), F(0), fake, fake, 16, 0, None) == 1
    # selftest: bad shapes
    assert L.fa4q_selftest_block_mma(fake, fake, fake, fake, 24, 64, 0, fake, None) == 2
    assert L.fa4q_selftest_block_mma(fake, fake, fake, fake, 128, 96, 0, fake, None) == 2


def test_binding_refuses_without_device(L):
    import torch
    import microscaled_fp4_flashattention_b200 as fa4q
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(RuntimeError):
        fa4q._stream()
