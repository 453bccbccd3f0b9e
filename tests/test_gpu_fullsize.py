"""Full-size parity: each measured workload in the launch configuration bench.py times
(one MoEForward per workload, workspace sized for its T, token tile chosen by the library).

Routing ids are compared bit-exactly for every token. Outputs are compared on a sample the
oracle can afford: 192 seeded random tokens, plus the tokens at both ends of the two most
loaded segments (their first and last 24 rows), which cover tile boundaries and ragged
tails. Tolerances as in tests/parity.py: BF16 |d| <= 2e-2 + 2^-8|ref| and rel-L2 <= 1e-2;
FP4 weights the element-wise bound derived from the layer's arithmetic and rel-L2 <= 3e-2.
"""
import functools

import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.parity import check_bf16, check_fp4_layer, oracle_bias, routing_kwargs, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = ["mixtral_prefill", "deepseek_decode", "deepseek_prefill", "mxfp4_decode", "mxfp4_prefill", "nvfp4",
        "mxfp4_w4a8_decode", "mxfp4_w4a8_prefill", "deepseek_decode_grouped"]


@functools.lru_cache(maxsize=2)
def _weights(E, B, B_used, H, I, wfmt, seed):
    """Weight sets depend only on these fields; decode and prefill of one family share them."""
    cfg = W.MoEConfig("w", T=1, H=H, I=I, E=E, topk=1, B=B, B_used=B_used, wfmt=wfmt, seed=seed)
    return W.gen_weights(cfg)


def _inputs(cfg):
    wg, wu, wd, src = _weights(cfg.E, cfg.B, cfg.B_used, cfg.H, cfg.I, cfg.wfmt, cfg.seed)
    extra = {"routing_bias": W.gen_routing_bias(cfg)} if cfg.routing == "deepseek_v3" else {}
    return W.MoEInputs(cfg, W.gen_x(cfg), W.gen_logits(cfg), src, wg, wu, wd, extra)


def _sample_tokens(cfg, perm, n_random=192, edge=24):
    g = np.random.default_rng(cfg.seed + 17)
    toks = set(g.choice(cfg.T, size=min(n_random, cfg.T), replace=False).tolist())
    lens = np.diff(np.concatenate([[0], perm["cu_seqlens"]]))
    for seg in np.argsort(-lens, kind="stable")[:2]:
        s1 = int(perm["cu_seqlens"][seg])
        s0 = s1 - int(lens[seg])
        rows = list(range(s0, min(s1, s0 + edge))) + list(range(max(s0, s1 - edge), s1))
        toks.update(int(perm["perm_token"][r]) for r in rows)
    return sorted(toks)


@pytest.mark.parametrize("name", FULL)
def test_fullsize_forward_matches_oracle(lib, name):
    cfg = W.CONFIGS[name]
    inp = _inputs(cfg)
    weights = [lib.Weight.from_host(w) for w in (inp.w_gate, inp.w_up, inp.w_down)]
    layer = lib.MoEForward(*weights, cfg.E, cfg.topk, cfg.B, to_dev(inp.replica_src) if cfg.B else None,
                           cfg.act, cfg.situ_alpha, cfg.situ_beta, cfg.act_quant, True, T_max=cfg.T,
                           **routing_kwargs(cfg, inp))
    ids = torch.empty(cfg.T, cfg.topk, dtype=torch.int32, device="cuda")
    out = layer(to_dev(inp.x), to_dev(inp.logits), topk_ids=ids)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    del layer, weights

    rids, _ = O.route(cfg, inp.logits.numpy(), oracle_bias(inp))
    assert np.array_equal(ids.cpu().numpy(), rids)
    perm = O.assign_rows(rids, cfg.E, cfg.B, inp.replica_src.numpy())
    toks = _sample_tokens(cfg, perm)
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, tokens=toks, routing_bias=oracle_bias(inp), keep=cfg.wfmt != "bf16")
    got = out[torch.tensor(toks, device="cuda")].float().cpu().numpy()
    if cfg.wfmt == "bf16":
        check_bf16(got, ref["out"], what=name)
    else:
        check_fp4_layer(got, ref, cfg, inp, what=name)
    torch.cuda.empty_cache()
