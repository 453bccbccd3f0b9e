"""Shared helpers of the GPU parity tests: tolerances and comparisons against the oracle.

Tolerances (written out in the tests that use them):
* indices (topk ids, cu_seqlens, perm_token, inv_perm, quantised codes): bit-exact;
* BF16 outputs: |gpu - ref| <= 2e-2 + 2^-8 |ref| elementwise and rel-L2 <= 1e-2. The 2^-8|ref|
  term is the bf16 rounding of the output itself (half an ulp is 2^-9|ref|; twice that leaves
  room for the bf16 rounding of the intermediate activation), which alone exceeds an absolute
  2e-2 at |ref| > 5;
* FP4-weight layers: rel-L2 <= 3e-2 against the oracle on the same dequantised weights.
* MXFP4-weight GEMMs stage the bf16 activations as two e4m3 terms with one e8m0 scale per
  32 values: every activation x is carried to within 1.07 * 2^-8 |x| + 2^(e-10), where
  2^e < 2 amax_b / 448 for the amax of its 32-value block. An output then lies within
  sum_k |W[n,k]| (0.0042 |x_k| + 5e-6 amax_b(k)) of the exact result, plus its own bf16
  rounding (mx8_staging_bound).
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


def mx8_staging_bound(a, ws, cu_seqlens, M_alloc):
    """Per-output bound of the MXFP4 GEMM's activation staging error (module docstring):
    sum_k |W_g[n,k]| * (0.0042 |a[r,k]| + 5e-6 amax of a[r]'s 32-value block holding k)."""
    from oracle import moe_oracle as O

    a = np.asarray(a, np.float64)
    M, K = a.shape
    amax = np.repeat(np.abs(a).reshape(M, K // 32, 32).max(axis=2), 32, axis=1)
    per = 0.0042 * np.abs(a) + 5e-6 * amax
    alpha = O.weight_alpha(ws)
    out = np.zeros((M_alloc, ws.N))
    for g, (s, e) in enumerate(O.segment_bounds(cu_seqlens)):
        if e > s:
            out[s:e] = alpha[g] * (per[s:e] @ np.abs(O.weight_rows(ws, g)).T)
    return out


def check_mx8(got, ref, bound, what=""):
    """|got - ref| <= staging bound + 2^-8 |ref| (the bf16 output) + 1e-6 max|ref|."""
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    lim = bound + 2.0 ** -8 * np.abs(ref) + 1e-6 * max(np.abs(ref).max(), 1e-30)
    worst = np.unravel_index(np.argmax(err - lim), err.shape) if err.size else None
    assert err.size == 0 or np.all(err <= lim), \
        f"{what}: max excess {np.max(err - lim):.3e} at {worst}: got {got[worst]} ref {ref[worst]}"
    return rel_l2(got, ref)


def routing_kwargs(cfg, inp):
    """MoEForward's routing arguments for a workload (the DeepSeekV3 method's bias on the GPU)."""
    bias = inp.extra.get("routing_bias")
    return dict(routing=cfg.routing, routing_bias=None if bias is None else to_dev(bias), n_group=cfg.n_group,
                topk_group=cfg.topk_group, routed_scaling_factor=cfg.routed_scaling_factor)


def oracle_bias(inp):
    """The DeepSeekV3 selection bias for the oracle, or None."""
    bias = inp.extra.get("routing_bias")
    return None if bias is None else bias.numpy()
