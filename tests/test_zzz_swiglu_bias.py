"""GPU parity of the per-expert GEMM biases and the SWIGLUOAI activation against the oracle:
the bias/activation row pass alone (moe_bias_act_and_mul), and the layer, which applies both
in the grouped GEMMs' epilogues.

Tolerances: the row pass computes in fp32 and rounds once to bf16, so each output lies within
half a bf16 ulp (<= 2^-8 |ref|) of the fp64 oracle plus the fp32 arithmetic's error (a few
fp32 ulps: <= 1e-6 |ref| + 1e-5, the absolute part for outputs that cancel); padding rows
are exactly zero. Layers: as in tests/parity.py
(BF16 |d| <= 2e-2 + 2^-8 |ref| and rel-L2 <= 1e-2; FP4 weights the element-wise bound derived
from the layer's arithmetic and rel-L2 <= 3e-2).

The file name sorts after every other test file: these kernels are the newest, so a run that
stops at its first failure has run all the others first.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.parity import check_bf16, check_fp4_layer, rel_l2, to_dev

pytestmark = pytest.mark.gpu

SEGS = [5, 0, 17, 1, 0, 40, 3]   # empty segments and lengths that are not multiples of anything
PAD = 3                           # rows past the last segment end: written as zero
I_COLS = 136                      # a multiple of 8 only

ACTS = {
    "silu": dict(act="silu"),
    "situ": dict(act="situ", situ_alpha=0.8, situ_beta=1.7),
    "swigluoai": dict(act="swigluoai", swiglu_alpha=1.702, swiglu_beta=1.0, swiglu_limit=1.5),
    "swigluoai_noclamp": dict(act="swigluoai", swiglu_alpha=0.9, swiglu_beta=-0.5, swiglu_limit=None),
}


def _oracle_act(gate, up, pw, p):
    return O.act_and_mul(gate, up, p["act"], p.get("situ_alpha", 1.0), p.get("situ_beta", 1.0), pw,
                         p.get("swiglu_alpha", 1.702), p.get("swiglu_beta", 1.0), p.get("swiglu_limit", 7.0))


@pytest.mark.parametrize("act", list(ACTS))
@pytest.mark.parametrize("in_f32,biases,weighted", [(True, "both", True), (False, "both", False),
                                                    (True, "gate", False), (False, "none", True)])
def test_bias_act_matches_oracle(lib, act, in_f32, biases, weighted):
    M, G = sum(SEGS) + PAD, len(SEGS)
    dt = torch.float32 if in_f32 else torch.bfloat16
    gate = W.gen_rows(M, I_COLS, seed=31, std=2.0, dtype=dt)
    up = W.gen_rows(M, I_COLS, seed=32, std=2.0, dtype=dt)
    bg = W.gen_rows(G, I_COLS, seed=33, std=0.5, dtype=torch.float32) if biases != "none" else None
    bu = W.gen_rows(G, I_COLS, seed=34, std=0.5, dtype=torch.float32) if biases == "both" else None
    pw = W.gen_rows(1, M, seed=35, dtype=torch.float32)[0].abs() if weighted else None
    cu = torch.tensor(np.cumsum(SEGS), dtype=torch.int32)
    p = ACTS[act]
    out = lib.moe_bias_act_and_mul(to_dev(gate), to_dev(up), to_dev(cu), to_dev(bg), to_dev(bu), to_dev(pw), **p)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)

    ref = np.zeros((M, I_COLS))
    g64, u64 = O.to_f64(gate), O.to_f64(up)
    for g, (s, e) in enumerate(O.segment_bounds(cu.numpy())):
        if e == s:
            continue
        gg = g64[s:e] + (O.to_f64(bg[g])[None, :] if bg is not None else 0.0)
        uu = u64[s:e] + (O.to_f64(bu[g])[None, :] if bu is not None else 0.0)
        ref[s:e] = _oracle_act(gg, uu, None if pw is None else O.to_f64(pw[s:e]), p)
    assert np.all(got[M - PAD:] == 0.0)
    err = np.abs(got - ref)
    lim = (2.0 ** -8 + 1e-6) * np.abs(ref) + 1e-5
    worst = np.unravel_index(np.argmax(err - lim), err.shape)
    assert np.all(err <= lim), f"max excess {np.max(err - lim):.3e} at {worst}: got {got[worst]} ref {ref[worst]}"
    if act == "swigluoai":     # the clamp was reached on both inputs
        assert np.abs(g64[:M - PAD]).max() > 1.5 and np.abs(u64[:M - PAD]).max() > 1.5


# Bias spreads are set near each layer's own magnitudes (gate/up projections ~0.3 for the
# BF16 weights, ~18 for MXFP4, ~60-80 for NVFP4; down outputs ~0.05, ~140, ~14 and ~1e5), so
# that leaving out either the gate/up or the down biases moves the output well past the
# tolerance (asserted on the oracle below).
SMALL = {
    # BF16 weights, SWIGLUOAI whose clamp the gate and up projections (std ~0.3) reach
    "bf16_swiglu_bias": W.MoEConfig("bf16_swiglu_bias", T=70, H=256, I=384, E=8, topk=2, act="swigluoai",
                                    swiglu_limit=0.3, bias=True, bias_down_std=0.03),
    # replicas and empty slots: every slot reads its own bias rows
    "bf16_silu_bias_replicas": W.MoEConfig("bf16_silu_bias_replicas", T=300, H=128, I=256, E=16, topk=4, B=6,
                                           B_used=4, logit_std=2.0, bias=True, bias_down_std=0.03),
    # SWIGLUOAI without biases
    "bf16_swiglu_nobias": W.MoEConfig("bf16_swiglu_nobias", T=40, H=128, I=192, E=8, topk=2, act="swigluoai",
                                      swiglu_alpha=1.2, swiglu_limit=None),
    # MXFP4 weights with bf16 activations, the GPT-OSS activation constants
    "mxfp4_swiglu_bias": W.MoEConfig("mxfp4_swiglu_bias", T=40, H=256, I=320, E=8, topk=4, act="swigluoai",
                                     wfmt="mxfp4", bias=True, bias_std=10.0, bias_down_std=100.0),
    # W4A8 (dynamic MXFP8 activations)
    "w4a8_swiglu_bias": W.MoEConfig("w4a8_swiglu_bias", T=40, H=256, I=320, E=8, topk=4, act="swigluoai",
                                    wfmt="mxfp4", act_quant=2, bias=True, bias_std=10.0, bias_down_std=100.0),
    # NVFP4 weights and activations, both GEMMs block-scaled
    "nvfp4_silu_bias": W.MoEConfig("nvfp4_silu_bias", T=50, H=512, I=256, E=16, topk=8, wfmt="nvfp4",
                                   act_quant=1, bias=True, bias_std=50.0, bias_down_std=1e5),
    # NVFP4 with gate/up staged in f16 (K = 272) and a SITU activation
    "nvfp4_situ_bias": W.MoEConfig("nvfp4_situ_bias", T=33, H=272, I=512, E=8, topk=4, wfmt="nvfp4",
                                   act_quant=1, act="situ", bias=True, bias_std=40.0, bias_down_std=10.0),
}

# Leaving out the gate/up or the down biases must move the oracle's output by at least this
# rel-L2 (over three times the loosest tolerance), so the comparison sees each of them.
BIAS_VISIBLE = 0.1


def _biases(inp):
    b = inp.extra.get("biases")
    return None if b is None else tuple(to_dev(t.float()) for t in b)


def _layer(lib, cfg, inp, **kw):
    dev = lambda ws: lib.Weight.from_host(ws)
    return lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, cfg.topk, cfg.B,
                          to_dev(inp.replica_src) if cfg.B else None, cfg.act, cfg.situ_alpha, cfg.situ_beta,
                          cfg.act_quant, kw.pop("apply_topk_in_fc1", True), T_max=cfg.T,
                          swiglu_alpha=cfg.swiglu_alpha, swiglu_beta=cfg.swiglu_beta,
                          swiglu_limit=cfg.swiglu_limit, biases=_biases(inp), **kw)


def _check(cfg, inp, out, ref, what):
    if cfg.wfmt == "bf16":
        check_bf16(out, ref["out"], what=what)
    else:
        check_fp4_layer(out, ref, cfg, inp, what=what)


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_swiglu_bias_matches_oracle(lib, name):
    cfg = SMALL[name]
    inp = W.gen_inputs(cfg)
    layer = _layer(lib, cfg, inp)
    ids = torch.empty(cfg.T, cfg.topk, dtype=torch.int32, device="cuda")
    out = layer(to_dev(inp.x), to_dev(inp.logits), topk_ids=ids)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, biases=inp.extra.get("biases"), keep=cfg.wfmt != "bf16")
    assert np.array_equal(ids.cpu().numpy(), ref["ids"])
    _check(cfg, inp, out, ref, name)
    b = inp.extra.get("biases")
    if b is not None:
        for part, bb in (("gate/up", (0 * b[0], 0 * b[1], b[2])), ("down", (b[0], b[1], 0 * b[2]))):
            alt = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                                inp.w_down, biases=bb)["out"]
            assert rel_l2(alt, ref["out"]) > BIAS_VISIBLE, f"{name}: the {part} biases barely matter"


def test_forward_bias_weight_in_combine(lib):
    # the route weight in the combine: the down bias is then weighted there with the rest
    cfg = SMALL["bf16_silu_bias_replicas"]
    inp = W.gen_inputs(cfg)
    layer = _layer(lib, cfg, inp, apply_topk_in_fc1=False)
    out = layer(to_dev(inp.x), to_dev(inp.logits))
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, apply_topk_in_fc1=False, biases=inp.extra["biases"])
    check_bf16(out, ref["out"], what="bias, weight in combine")


def test_forward_bias_input_weight_top1(lib):
    # a given top-1 with weights in [0.1, 2] on the input: the experts see x * w, and neither
    # the activation nor the biases take the weight again
    cfg = W.MoEConfig("bias_top1", T=90, H=128, I=192, E=8, topk=1, act="swigluoai", swiglu_limit=0.3, bias=True,
                      bias_down_std=0.03)
    inp = W.gen_inputs(cfg)
    g = np.random.default_rng(3)
    gid = g.integers(0, cfg.E, (cfg.T, 1)).astype(np.int32)
    gw = g.uniform(0.1, 2.0, (cfg.T, 1)).astype(np.float32)
    layer = _layer(lib, cfg, inp, routing="given", apply_router_weight_on_input=True)
    out = layer(to_dev(inp.x), None, topk_ids_in=to_dev(torch.from_numpy(gid)), topk_w_in=to_dev(torch.from_numpy(gw)))
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.moe_forward(cfg, inp.x, None, inp.replica_src.numpy(), inp.w_gate, inp.w_up, inp.w_down,
                        given_topk=(gid, gw), apply_router_weight_on_input=True, biases=inp.extra["biases"])
    check_bf16(out, ref["out"], what="bias, input weight")


@pytest.mark.slow
def test_fullsize_swiglu_bias_decode(lib):
    # the MXFP4 decode workload (T=32, H=I=2880, E=128, top-4) with SWIGLUOAI and biases in
    # the launch configuration bench.py times, every token compared
    cfg = W.CONFIGS["mxfp4_swiglu_bias_decode"]
    inp = W.gen_inputs(cfg)
    layer = _layer(lib, cfg, inp)
    out = layer(to_dev(inp.x), to_dev(inp.logits))
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, biases=inp.extra["biases"], keep=True)
    _check(cfg, inp, out, ref, cfg.name)


@pytest.mark.slow
def test_fullsize_swiglu_bias_prefill(lib):
    # the MXFP4 prefill workload (T=4096) with SWIGLUOAI and biases as bench.py times it;
    # ids for every token, outputs on the full-size tests' token sample
    from tests.test_gpu_fullsize import _sample_tokens

    cfg = W.CONFIGS["mxfp4_swiglu_bias_prefill"]
    inp = W.gen_inputs(cfg)
    layer = _layer(lib, cfg, inp)
    ids = torch.empty(cfg.T, cfg.topk, dtype=torch.int32, device="cuda")
    out = layer(to_dev(inp.x), to_dev(inp.logits), topk_ids=ids)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    rids, _ = O.route(cfg, inp.logits.numpy())
    assert np.array_equal(ids.cpu().numpy(), rids)
    toks = _sample_tokens(cfg, O.assign_rows(rids, cfg.E, cfg.B, inp.replica_src.numpy()))
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, tokens=toks, biases=inp.extra["biases"], keep=True)
    got = out[torch.tensor(toks, device="cuda")].float().cpu().numpy()
    check_fp4_layer(got, ref, cfg, inp, what=cfg.name)
