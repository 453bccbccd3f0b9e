"""Seeded synthetic workloads for the fused MoE expert layer.

This module only draws random inputs. It holds none of the layer's arithmetic:
no routing, no permutation, no GEMM, no activation and no quantisation rule.
Both the CPU oracle (``oracle/``) and the CUDA library's tests and benchmark
take their inputs from here, so that the two sides see identical bits.

Every tensor has its own ``torch.Generator`` seeded from ``(seed, stream id)``,
so drawing one tensor never shifts the bits of another, and a caller that only
needs ``x`` does not pay for the weights.

Shapes and distributions follow the workloads the pages describe:

* the MoonEP experts page (``vllm...experts.moonep_experts``, module docstring)
  fixes the layout: ``x [T,H]``, gate/up ``[E+B, I, H]``, down ``[E+B, H, I]``,
  with rows ``[E, E+B)`` being redundant copies of hot experts;
* the TRTLLM MXFP4 page (``...experts.trtllm_mxfp4_moe``,
  ``TrtLlmMxfp4ExpertsBase``) fixes MXFP4 weights (e2m1 codes, e8m0 scale per
  32 values along K) and the SITU activation;
* the DeepSeek-V4 FlashInfer page (``vllm.models.deepseek_v4.nvidia.fi_moe``,
  ``_realloc_nvfp4_params``) fixes the NVFP4 layout: e2m1 codes, fp8-e4m3
  scale per 16 values along K, one fp32 ``weight_scale_2`` per expert for gate,
  up and down separately.

Packed FP4 codes hold two values per byte, the even-K value in the low nibble.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import torch

# Stream ids: one independent generator per drawn tensor.
_S_X, _S_LOGITS, _S_GATE, _S_UP, _S_DOWN, _S_REPLICA = 1, 2, 3, 4, 5, 6
_S_GATE_SCALE, _S_UP_SCALE, _S_DOWN_SCALE = 7, 8, 9
_S_GATE_ALPHA, _S_UP_ALPHA, _S_DOWN_ALPHA = 10, 11, 12
_S_BIAS = 13

WFMT_BF16, WFMT_MXFP4, WFMT_NVFP4 = "bf16", "mxfp4", "nvfp4"


@dataclass(frozen=True)
class MoEConfig:
    """One workload: problem sizes plus the distributions its inputs are drawn from."""

    name: str
    T: int                     # tokens
    H: int                     # hidden size (K of gate/up, N of down)
    I: int                     # intermediate size (N of gate/up, K of down)
    E: int                     # routed experts
    topk: int
    B: int = 0                 # redundant expert slots appended after the E experts
    B_used: int = 0            # how many of the B slots receive tokens
    act: str = "silu"          # "silu" (silu(gate)*up) or "situ"
    situ_alpha: float = 1.0    # SITU gate cap  (activation_situ_beta)
    situ_beta: float = 1.0     # SITU up cap    (activation_situ_linear_beta)
    wfmt: str = WFMT_BF16
    act_quant: int = 0         # 1 = dynamic NVFP4, 2 = dynamic MXFP8 quantisation of activations
    routing: str = "renormalize"   # or "deepseek_v3": grouped top-k on sigmoid scores
    swiglu_alpha: float = 1.702        # SWIGLUOAI parameters (act = "swigluoai")
    swiglu_beta: float = 1.0
    swiglu_limit: float | None = 7.0
    bias: bool = False                 # per-row GEMM biases (gemm1_bias, gemm2_bias)
    bias_std: float = 0.1              # their spread: gate and up, and down
    bias_down_std: float = 0.1
    n_group: int = 1
    topk_group: int = 1
    routed_scaling_factor: float = 1.0
    x_std: float = 1.0
    logit_std: float = 1.0
    w_std: float = 0.02
    mx_exp_lo: int = -8        # MXFP4 scale exponents drawn uniformly from [lo, hi]
    mx_exp_hi: int = 0
    nv_scale_lo: float = 0.25  # NVFP4 block scales drawn from U[lo, hi], rounded to e4m3
    nv_scale_hi: float = 2.0
    alpha_lo: float = 0.5      # NVFP4 weight_scale_2 drawn from U[lo, hi] per expert
    alpha_hi: float = 1.5
    seed: int = 0

    @property
    def G(self) -> int:
        """Weight rows: experts plus redundant slots."""
        return self.E + self.B

    @property
    def NvS(self) -> int:
        """Routed (token, expert) pairs: rows of the expert-contiguous activations."""
        return self.T * self.topk

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)


# The workloads. "tiny" is the small parity case; the others are the measured shapes.
CONFIGS: dict[str, MoEConfig] = {
    "tiny": MoEConfig("tiny", T=16, H=128, I=256, E=8, topk=2),
    "mixtral_prefill": MoEConfig("mixtral_prefill", T=4096, H=4096, I=14336, E=8, topk=2),
    "deepseek_decode": MoEConfig("deepseek_decode", T=64, H=7168, I=2048, E=256, topk=8,
                                 B=16, B_used=8, logit_std=2.0),
    "deepseek_prefill": MoEConfig("deepseek_prefill", T=8192, H=7168, I=2048, E=256, topk=8,
                                  B=16, B_used=8, logit_std=2.0),
    "mxfp4_decode": MoEConfig("mxfp4_decode", T=32, H=2880, I=2880, E=128, topk=4,
                              act="situ", wfmt=WFMT_MXFP4),
    "mxfp4_prefill": MoEConfig("mxfp4_prefill", T=4096, H=2880, I=2880, E=128, topk=4,
                               act="situ", wfmt=WFMT_MXFP4),
    "nvfp4": MoEConfig("nvfp4", T=1024, H=7168, I=2048, E=256, topk=8,
                       wfmt=WFMT_NVFP4, act_quant=1),
    # DeepSeekV3 routing on the DeepSeek decode shape: 8 groups of 32, 4 kept, scaling 2.5
    "deepseek_decode_grouped": MoEConfig("deepseek_decode_grouped", T=64, H=7168, I=2048, E=256, topk=8,
                                         B=16, B_used=8, logit_std=2.0, routing="deepseek_v3", n_group=8,
                                         topk_group=4, routed_scaling_factor=2.5),
    # the W4A8 mode of the MXFP4 experts: the MXFP4 shapes with dynamic MXFP8 activations
    # the MXFP4 shapes with SWIGLUOAI (GPT-OSS constants) and per-expert GEMM biases, spread
    # near the projections' own magnitudes (gate/up ~18, down ~400 with these weights)
    "mxfp4_swiglu_bias_decode": MoEConfig("mxfp4_swiglu_bias_decode", T=32, H=2880, I=2880, E=128, topk=4,
                                          act="swigluoai", wfmt=WFMT_MXFP4, bias=True, bias_std=10.0,
                                          bias_down_std=400.0),
    "mxfp4_swiglu_bias_prefill": MoEConfig("mxfp4_swiglu_bias_prefill", T=4096, H=2880, I=2880, E=128, topk=4,
                                           act="swigluoai", wfmt=WFMT_MXFP4, bias=True, bias_std=10.0,
                                           bias_down_std=400.0),
    "mxfp4_w4a8_decode": MoEConfig("mxfp4_w4a8_decode", T=32, H=2880, I=2880, E=128, topk=4,
                                   act="situ", wfmt=WFMT_MXFP4, act_quant=2),
    "mxfp4_w4a8_prefill": MoEConfig("mxfp4_w4a8_prefill", T=4096, H=2880, I=2880, E=128, topk=4,
                                    act="situ", wfmt=WFMT_MXFP4, act_quant=2),
}


def _gen(cfg: MoEConfig, stream: int) -> torch.Generator:
    return torch.Generator().manual_seed(cfg.seed * 1_000_003 + stream)


def gen_x(cfg: MoEConfig) -> torch.Tensor:
    """Hidden states ``x [T,H]`` bf16, drawn N(0, x_std^2) in fp32 and rounded to bf16."""
    g = _gen(cfg, _S_X)
    return (torch.randn(cfg.T, cfg.H, generator=g) * cfg.x_std).to(torch.bfloat16)


def gen_logits(cfg: MoEConfig) -> torch.Tensor:
    """Router logits ``[T,E]`` fp32, N(0, logit_std^2)."""
    g = _gen(cfg, _S_LOGITS)
    return torch.randn(cfg.T, cfg.E, generator=g) * cfg.logit_std


def gen_routing_bias(cfg: MoEConfig) -> torch.Tensor:
    """Selection bias of the DeepSeekV3 routing (e_score_correction_bias) ``[E]`` fp32,
    N(0, 0.05^2): of the order of the spread of sigmoid scores near 0.5, so it reorders
    close candidates without deciding most choices."""
    g = _gen(cfg, _S_BIAS)
    return torch.randn(cfg.E, generator=g) * 0.05


def gen_biases(cfg: MoEConfig) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Per-row GEMM biases: gate and up ``[G,I]`` fp32 N(0, bias_std^2), down ``[G,H]`` fp32
    N(0, bias_down_std^2); ``gen_inputs`` makes replica slots copy their source expert's."""
    g = _gen(cfg, _S_BIAS + 1)
    G = cfg.E + cfg.B
    bg = torch.randn(G, cfg.I, generator=g) * cfg.bias_std
    bu = torch.randn(G, cfg.I, generator=g) * cfg.bias_std
    bd = torch.randn(G, cfg.H, generator=g) * cfg.bias_down_std
    return bg, bu, bd


def gen_replica_src(cfg: MoEConfig) -> torch.Tensor:
    """Source expert of every redundant slot, ``[B]`` int32.

    ``B_used`` distinct experts are drawn; slot ``s < B_used`` is a used replica
    of ``src[s]``. The remaining slots also hold copies of drawn experts (their
    weights exist) but receive no tokens and are marked -1.
    Returns ``(replica_src [B] int32 with -1 for unused, copy_of [B] int64)``.
    """
    if cfg.B == 0:
        return torch.zeros(0, dtype=torch.int32), torch.zeros(0, dtype=torch.int64)
    g = _gen(cfg, _S_REPLICA)
    copy_of = torch.randperm(cfg.E, generator=g)[: cfg.B].to(torch.int64)
    src = copy_of.clone().to(torch.int32)
    src[cfg.B_used:] = -1
    return src, copy_of


@dataclass
class WeightSet:
    """One projection's weights in the layer's canonical (checkpoint) layout.

    ``data``: bf16 ``[G,N,K]`` or uint8 packed e2m1 ``[G,N,K/2]`` (even K in the low nibble).
    ``scale``: None, uint8 e8m0 ``[G,N,K/32]`` (MXFP4) or uint8 e4m3 ``[G,N,K/16]`` (NVFP4).
    ``alpha``: None or fp32 ``[G]`` per-expert global scale (NVFP4 ``weight_scale_2``).
    """

    fmt: str
    data: torch.Tensor
    scale: torch.Tensor | None = None
    alpha: torch.Tensor | None = None

    @property
    def G(self) -> int:
        return self.data.shape[0]

    @property
    def N(self) -> int:
        return self.data.shape[1]

    @property
    def K(self) -> int:
        return self.data.shape[2] * (2 if self.fmt != WFMT_BF16 else 1)


def _expand_replicas(t: torch.Tensor, cfg: MoEConfig, copy_of: torch.Tensor) -> torch.Tensor:
    """Append the B redundant slots, each an exact copy of its source expert."""
    if cfg.B == 0:
        return t
    return torch.cat([t, t[copy_of]], dim=0)


def _gen_one(cfg: MoEConfig, N: int, K: int, s_data: int, s_scale: int, s_alpha: int,
             copy_of: torch.Tensor) -> WeightSet:
    E = cfg.E
    if cfg.wfmt == WFMT_BF16:
        g = _gen(cfg, s_data)
        out = torch.empty(E, N, K, dtype=torch.bfloat16)
        for e in range(E):  # per expert: bounded fp32 temporaries
            out[e] = (torch.randn(N, K, generator=g) * cfg.w_std).to(torch.bfloat16)
        return WeightSet(WFMT_BF16, _expand_replicas(out, cfg, copy_of))
    if K % 2:
        raise ValueError("FP4 weights need an even K")
    g = _gen(cfg, s_data)
    # Every byte holds two independent codes, each uniform over the 16 e2m1 codes.
    data = torch.randint(0, 256, (E, N, K // 2), generator=g, dtype=torch.uint8)
    gs = _gen(cfg, s_scale)
    if cfg.wfmt == WFMT_MXFP4:
        if K % 32:
            raise ValueError("MXFP4 needs K % 32 == 0")
        exp = torch.randint(cfg.mx_exp_lo, cfg.mx_exp_hi + 1, (E, N, K // 32), generator=gs)
        scale = (exp + 127).to(torch.uint8)  # e8m0 biased exponent
        alpha = None
    elif cfg.wfmt == WFMT_NVFP4:
        if K % 16:
            raise ValueError("NVFP4 needs K % 16 == 0")
        u = torch.rand(E, N, K // 16, generator=gs) * (cfg.nv_scale_hi - cfg.nv_scale_lo) + cfg.nv_scale_lo
        scale = u.to(torch.float8_e4m3fn).view(torch.uint8)
        ga = _gen(cfg, s_alpha)
        alpha = torch.rand(E, generator=ga) * (cfg.alpha_hi - cfg.alpha_lo) + cfg.alpha_lo
    else:
        raise ValueError(f"unknown weight format {cfg.wfmt}")
    return WeightSet(cfg.wfmt,
                     _expand_replicas(data, cfg, copy_of),
                     _expand_replicas(scale, cfg, copy_of),
                     None if alpha is None else _expand_replicas(alpha, cfg, copy_of).contiguous())


@dataclass
class MoEInputs:
    cfg: MoEConfig
    x: torch.Tensor
    logits: torch.Tensor
    replica_src: torch.Tensor
    w_gate: WeightSet
    w_up: WeightSet
    w_down: WeightSet
    extra: dict = field(default_factory=dict)


def gen_weights(cfg: MoEConfig) -> tuple[WeightSet, WeightSet, WeightSet, torch.Tensor]:
    src, copy_of = gen_replica_src(cfg)
    wg = _gen_one(cfg, cfg.I, cfg.H, _S_GATE, _S_GATE_SCALE, _S_GATE_ALPHA, copy_of)
    wu = _gen_one(cfg, cfg.I, cfg.H, _S_UP, _S_UP_SCALE, _S_UP_ALPHA, copy_of)
    wd = _gen_one(cfg, cfg.H, cfg.I, _S_DOWN, _S_DOWN_SCALE, _S_DOWN_ALPHA, copy_of)
    return wg, wu, wd, src


def gen_inputs(cfg: MoEConfig) -> MoEInputs:
    """All inputs of one workload, on the CPU."""
    wg, wu, wd, src = gen_weights(cfg)
    extra = {"routing_bias": gen_routing_bias(cfg)} if cfg.routing == "deepseek_v3" else {}
    if cfg.bias:
        bg, bu, bd = gen_biases(cfg)
        for s, e in enumerate(src.tolist()):   # a replica slot holds its source expert's biases
            if e >= 0:
                bg[cfg.E + s], bu[cfg.E + s], bd[cfg.E + s] = bg[e], bu[e], bd[e]
        extra["biases"] = (bg, bu, bd)
    return MoEInputs(cfg, gen_x(cfg), gen_logits(cfg), src, wg, wu, wd, extra)


def gen_grouped_gemm_case(M_alloc: int, seg_lens: list[int], N: int, K: int, seed: int = 0,
                          a_std: float = 1.0, w_std: float = 0.02):
    """A standalone grouped-GEMM case: activations ``[M_alloc,K]`` bf16, weights ``[G,N,K]`` bf16
    and the segment lengths (their running sum is the caller's business)."""
    g = torch.Generator().manual_seed(seed)
    a = (torch.randn(M_alloc, K, generator=g) * a_std).to(torch.bfloat16)
    w = (torch.randn(len(seg_lens), N, K, generator=g) * w_std).to(torch.bfloat16)
    return a, w, torch.tensor(seg_lens, dtype=torch.int32)


def gen_rows(R: int, K: int, seed: int = 0, std: float = 1.0, dtype=torch.bfloat16) -> torch.Tensor:
    """Generic seeded rows ``[R,K]`` (activation-quant and activation cases)."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(R, K, generator=g) * std).to(dtype)
