"""The bounded-wait path of the grouped GEMMs on a B200.

Every pipeline wait in the GEMM kernels gives up after a cycle limit (about one second by
default), records MOE_ERR_TIMEOUT in the workspace's error word, stops every role of the
CTA, lets the copies and MMAs already in flight finish, frees tensor memory and returns.
MOE_WAIT_LIMIT_CYCLES shortens the limit for a launch; at one cycle the first wait that
does not succeed at once gives up. Each case checks that the forward returns, that the
error word reads MOE_ERR_TIMEOUT, and that the next forward on the same workspace, with the
default limit, matches the oracle. Nothing here faults or hangs the GPU: the waits that
give up end in the kernel's own orderly exit.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.parity import check_bf16, check_fp4_layer, to_dev

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 7

CASES = {
    # one per GEMM kernel: BF16 on one SM; NVFP4 x NVFP4 block-scaled; MXFP4 x e4m3 hi/lo;
    # NVFP4 weights with bf16 activations (converter warps into tensor memory)
    "bf16": W.MoEConfig("t_bf16", T=300, H=512, I=256, E=8, topk=2),
    "nvfp4": W.MoEConfig("t_nvfp4", T=50, H=512, I=256, E=16, topk=8, wfmt="nvfp4", act_quant=1),
    "mxfp4": W.MoEConfig("t_mxfp4", T=40, H=256, I=320, E=8, topk=4, act="situ", wfmt="mxfp4"),
    "nvfp4_a16": W.MoEConfig("t_nvfp4_a16", T=50, H=512, I=256, E=16, topk=8, wfmt="nvfp4"),
    # BF16 on CTA pairs (segments of about 150 rows), with the token rows pre-gathered or
    # gathered by the GEMM's producer warp
    "bf16_pairs": W.MoEConfig("t_bf16_pairs", T=600, H=256, I=256, E=8, topk=2),
    "bf16_pairs_gather": W.MoEConfig("t_bf16_pairs_gather", T=600, H=256, I=256, E=8, topk=2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_wait_timeout_is_reported_and_the_next_call_is_correct(lib, name, monkeypatch):
    cfg = CASES[name]
    inp = W.gen_inputs(cfg)
    dev = lambda ws: lib.Weight.from_host(ws)
    layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, cfg.topk, act=cfg.act,
                           situ_alpha=cfg.situ_alpha, situ_beta=cfg.situ_beta, act_quant=cfg.act_quant,
                           T_max=cfg.T)
    x, logits = to_dev(inp.x), to_dev(inp.logits)
    monkeypatch.setenv("MOE_GEMM_PAIRS", "1" if name.startswith("bf16_pairs") else "0")
    monkeypatch.setenv("MOE_FUSED_GATHER", "1" if name == "bf16_pairs_gather" else "0")
    monkeypatch.setenv("MOE_WAIT_LIMIT_CYCLES", "1")
    layer(x, logits)
    torch.cuda.synchronize()                       # the kernels returned
    assert layer.device_error() == MOE_ERR_TIMEOUT
    monkeypatch.delenv("MOE_WAIT_LIMIT_CYCLES")
    out = layer(x, logits)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, keep=cfg.wfmt != "bf16")
    if cfg.wfmt == "bf16":
        check_bf16(out, ref["out"], what=name)
    else:
        check_fp4_layer(out, ref, cfg, inp, what=name)
