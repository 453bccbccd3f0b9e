"""Shared helpers of the GPU parity tests: tolerances and comparisons against the oracle.

Tolerances (written out in the tests that use them):
* indices (topk ids, cu_seqlens, perm_token, inv_perm, quantised codes): bit-exact;
* BF16 outputs: |gpu - ref| <= 2e-2 + 2^-8 |ref| elementwise and rel-L2 <= 1e-2. The 2^-8|ref|
  term is the bf16 rounding of the output itself (half an ulp is 2^-9|ref|; twice that leaves
  room for the bf16 rounding of the intermediate activation), which alone exceeds an absolute
  2e-2 at |ref| > 5;
* FP4-weight layers: rel-L2 <= 3e-2 against the oracle on the same dequantised weights.
"""
import numpy as np
import torch

BF16_ATOL = 2e-2
BF16_RTOL = 2.0 ** -8
BF16_REL_L2 = 1e-2
FP4_REL_L2 = 3e-2


def to_dev(t):
    return None if t is None else t.cuda().contiguous()


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def check_bf16(got, ref, atol=BF16_ATOL, rtol=BF16_RTOL, rel=BF16_REL_L2, what=""):
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape) if err.size else None
    assert err.size == 0 or np.all(err <= bound), \
        f"{what}: max excess {np.max(err - bound):.3e} at {worst}: got {got[worst]} ref {ref[worst]}"
    r = rel_l2(got, ref)
    assert r <= rel, f"{what}: rel-L2 {r:.3e} > {rel}"
    return float(np.max(err)) if err.size else 0.0, r
