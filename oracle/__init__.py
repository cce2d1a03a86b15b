"""CPU oracle for fused 4-bit microscaled FlashAttention.

TEST INFRASTRUCTURE ONLY.  Only the tests, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` may import this package.
The CUDA library never calls it, and it shares no code with the CUDA path.

A plain, slow, obviously-correct numpy implementation, written from the pages:

* `formats`   - E2M1 elements, UE4M3 and UE8M0 scales, NVFP4 / MXFP4 block
                quantisation with the optional scale bound Qmax (UOS) and the
                optional Smooth-QK multiplier.
* `attention` - tiled online-softmax attention with pre-normalisation
                quantisation of the exponentials (PNQ) and the normaliser taken
                from the quantised P_hat (P-Reordering); plain FP64 attention.
* `decode`    - softmax attention of one query over an FP4 paged KV cache
                plus a BF16 vertical-line set and window.
* `smooth`    - the calibration of the static per-channel Q/K multipliers.
* `hyquant`   - vertical-line identification by accumulated column mass
                (diagnostic; not on the timed path).
* `rotate`    - Hadamard rotation of Q and K rows before quantisation (the
                outlier-spreading alternative to Smooth-QK; an ablation).
* `hybrid`    - hybrid-precision prefill: vertical-line and window keys in BF16,
                the rest FP4, one online softmax.
* `bitdecode` - decode with a dual-residual FP4 query and FP4 probabilities against
                the FP4 paged cache.
* `report_accuracy` - (run by hand) the method's error against unquantised attention on
                the synthetic workloads, from the oracle alone.

Every function states the passage it follows.  Floating point is FP64 except
where the method fixes FP32 decisions (scale selection and element rounding),
which are taken in IEEE FP32 exactly as specified in `formats`.

Parity status: `formats`, `attention`, `decode`, `smooth`, `rotate`, `hybrid` and `bitdecode`
are pinned by the
`-m "not gpu"` tests in `tests/test_oracle_*.py`.  `hyquant` is a diagnostic
pinned only qualitatively (planted vertical lines are recovered).
"""
from . import formats, attention, decode, smooth, hyquant, rotate, hybrid, bitdecode  # noqa: F401
